"""fp64 CPU oracle for the Ideogram 4 DiT block hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``, never by the ``joint_attention_block_b200``
package.  It shares no code with the CUDA path.
"""
from .ideogram4 import (  # noqa: F401
    attention,
    bf16_to_f64,
    cond_proj_forward,
    denoise_steps,
    dequant,
    dit_block_forward,
    dit_stack_forward,
    e4m3_round,
    e4m3_to_f64,
    euler_cfg_step,
    f64_to_bf16_bits,
    gelu,
    inv_freq,
    mrope,
    mrope_angles,
    mrope_positions,
    qk_e4m3_scale,
    quantize_qk,
    quantize_rows_act,
    rmsnorm,
)
