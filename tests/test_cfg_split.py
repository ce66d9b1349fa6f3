"""The two-rank CFG-branch split on CPU: two gloo ranks run the conditional and the unconditional
branch with the oracle as their compute, exchange velocities once per step, and must end with
the latent the single-process oracle composition gives (and the same latent on both ranks).
A rank that fails before its exchange makes the other rank's collective end with an error."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from types import SimpleNamespace


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg():
    return SimpleNamespace(d_model=8, n_heads=2, head_dim=4, d_mlp=16, rope_sections=(1, 0, 1), rope_theta=10000.0,
                           eps=1e-6, gelu_tanh=0)


def _problem():
    from joint_attention_block_b200 import synth

    cfg = _cfg()
    r = np.random.default_rng(70)

    def weights(seed):
        rr = np.random.default_rng(seed)
        w = {}
        for name, shape in (("w_qkv", (24, 8)), ("w_o", (8, 8)), ("w_up", (16, 8)), ("w_down", (8, 16))):
            w[name], w["s_" + name[2:]] = synth.quantize_rows_e4m3(rr.standard_normal(shape).astype(np.float32) * 0.3)
        for name, n in (("g_norm1", 8), ("g_norm2", 8), ("g_q", 4), ("g_k", 4)):
            w[name] = synth.to_bf16_bits(1.0 + 0.1 * rr.standard_normal(n))
        return w

    wc = [weights(71), weights(72)]
    wu = [weights(73), weights(74)]
    z0 = r.standard_normal((1, 6, 8))
    tc = synth.to_bf16_bits(r.standard_normal((1, 3, 8)))
    tu = synth.to_bf16_bits(np.zeros((1, 2, 8)))
    return cfg, wc, wu, z0, tc, tu, [7.0, 7.0, 3.0], [-0.25, -0.25, -0.5]


def _rank_main(rank, port, out, fail_rank):
    import torch.distributed as dist

    import oracle
    from joint_attention_block_b200.cfg_split import SplitStep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=10))
    try:
        if rank == fail_rank:
            raise SystemExit(3)  # this rank dies before its first exchange
        cfg, wc, wu, z0, tc, tu, gws, dts = _problem()
        gh, gw = 2, 3

        def branch_velocity(z, branch):
            zb = oracle.f64_to_bf16_bits(z.numpy())
            text, ws = (tc, wc) if branch == 0 else (tu, wu)
            x = np.concatenate([text, zb], axis=1)
            v = oracle.f64_to_bf16_bits(oracle.dit_stack_forward(cfg, ws, x, text.shape[1], gh, gw)[:, text.shape[1]:])
            return torch.from_numpy(v.view(np.int16).copy())

        def update(z, v_c, v_u, g, dt):
            vc = v_c.numpy().view(np.uint16)
            vu = v_u.numpy().view(np.uint16)
            z.copy_(torch.from_numpy(oracle.euler_cfg_step(z.numpy(), vc, vu, g, dt)))

        z = torch.from_numpy(z0.copy())
        SplitStep().run(z, branch_velocity, update, gws, dts)
        out.put((rank, "ok", z.numpy()))
    except SystemExit:
        out.put((rank, "died", None))
        out.close()
        out.join_thread()  # flush the report before the hard exit
        os._exit(3)
    except Exception as e:  # the surviving rank's collective fails
        out.put((rank, "error", f"{type(e).__name__}: {e}"))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def _run(fail_rank):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q, fail_rank)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, status, val = q.get(timeout=180)
        res[rank] = (status, val)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return res, [p.exitcode for p in procs]


def test_split_step_equals_the_single_process_composition():
    import oracle

    res, codes = _run(fail_rank=-1)
    assert codes == [0, 0]
    cfg, wc, wu, z0, tc, tu, gws, dts = _problem()
    want = oracle.denoise_steps(cfg, wc, wu, tc, tu, z0, 2, 3, gws, dts)
    for rank in (0, 1):
        status, z = res[rank]
        assert status == "ok", z
        assert np.array_equal(z, want), f"rank {rank}"


def test_a_rank_that_dies_makes_the_other_fail_not_hang():
    res, codes = _run(fail_rank=1)
    assert res[1][0] == "died"
    assert res[0][0] == "error", res[0]


def test_split_needs_two_ranks():
    import torch.distributed as dist

    from joint_attention_block_b200.cfg_split import SplitStep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        with pytest.raises(ValueError):
            SplitStep()
    finally:
        dist.destroy_process_group()
