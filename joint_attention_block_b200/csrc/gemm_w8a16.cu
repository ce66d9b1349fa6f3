// Y = act( A (W8)^T * scale ) + R on the 5th-generation tensor cores.
//
// A: 16-bit activations [M, K] row-major (M = tokens).  W8: e4m3 weights [N, K]
// row-major with an fp32 per-output-row scale, the storage of the Ideogram 4 FP8
// checkpoint (unsloth diffusion_ideogram4.py commit log, fp8 loader commit: the real
// weight is fp8 * weight_scale[:, None]).
//
// The checkpoint's numerics are W8 dequantised, activations 16-bit.  e4m3 is a
// subset of both bf16 and f16, so the weights are widened on chip, exactly, to the
// activation format and fed to tcgen05.mma kind::f16 with an fp32 accumulator; the
// per-row scale is applied once per output in the epilogue (scale[n] * sum_k a*w8
// is sum_k a*(w8*scale[n]) up to rounding).
//
// The GEMM is bound by the stream of tiles from L2, so the tile is shaped for bytes
// per FLOP.  Two CTAs on two SMs (a cluster of 2) share one 256 (tokens) x 512
// (channels) tile through the pair form of the MMA (tcgen05.mma.cta_group::2,
// M = 256, N = 256, issued twice per K-step into two TMEM accumulators): each
// activation tile is reused for 512 channels and each weight tile for 256 tokens,
// 256 FLOP per L2 byte.  Each CTA TMA-loads its own 128 tokens (half of A) and its
// own 2 x 128 e4m3 weight rows (its half of each B), widens those rows into a
// 128B-swizzled K-major tile in its shared memory, and receives 128 tokens x 512
// channels of D in its TMEM (all 512 columns).  Both CTAs' activation loads count
// on the leader's barrier, both CTAs' converter warps arrive on the leader's
// barrier, and the leader's MMA commits arrive on both CTAs' barriers.  No TMA load
// is multicast.
//
// Per CTA (grid.z = K splits):
//   warp 0      TMA producer: 128 x 64 activations (128B swizzle) and 2 x (128 x 64
//               bytes) e4m3 weights (64B swizzle) per stage, 3-stage ring.
//   warp 1      TMEM allocation (pair); in the leader, one lane issues 2 x 4 pair
//               MMAs per stage.
//   warps 2..9  converters: thread = one weight row; widen 64 e4m3 bytes to f16 (or
//               bf16) and store them into the 2-stage widened ring.  Then the
//               epilogue: thread = one token row of TMEM (warp w reads lanes
//               32*(w%4).., accumulator (w-2)/4), scale, optional GELU; then, through
//               shared memory, row-major: optional residual, 16-bit or fp32 stores
//               that fill whole sectors.
#include <string.h>

#include "common.cuh"

namespace jab {
namespace gemm {

constexpr int BM = 256;      // tokens per pair tile (MMA M over the pair)
constexpr int BM_CTA = 128;  // tokens each CTA loads (its TMEM lanes)
constexpr int BN = 512;      // output channels per pair tile: two MMAs of N = 256
constexpr int BN_MMA = 256;
constexpr int BK = 64;
constexpr int RAW_STAGES = 3;
constexpr int CVT_STAGES = 2;
constexpr int X_BYTES = BM_CTA * BK * 2;   // TMA box {BK, 128} of 16-bit activations
constexpr int W8_BLOCK = 128 * BK;         // TMA box {BK, 128} of e4m3 bytes (64B swizzle)
constexpr int W8_BYTES = 2 * W8_BLOCK;
constexpr int W16_BLOCK = 128 * BK * 2;    // 128 widened rows, 128B-swizzled K-major
constexpr int W16_BYTES = 2 * W16_BLOCK;
constexpr int THREADS = 320;
constexpr int CVT_WARPS = 8;
constexpr int TMEM_COLS = 512;
constexpr int MAX_PAIRS = 74;  // 148 SMs / 2

constexpr int OFF_X = 0;
constexpr int OFF_W8 = OFF_X + RAW_STAGES * X_BYTES;
constexpr int OFF_W16 = OFF_W8 + RAW_STAGES * W8_BYTES;
constexpr int OFF_SCALE = OFF_W16 + CVT_STAGES * W16_BYTES;
constexpr int OFF_BAR = OFF_SCALE + BN * 4;
constexpr int NUM_BARS = 3 * RAW_STAGES + 2 * CVT_STAGES + 2 + 2 * CVT_WARPS;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
// Epilogue boxes: per epilogue warp two output boxes and two residual boxes of 32 tokens x 32
// channels (up to fp32: 4 KB each), placed in the rings, which are free by then.
constexpr int EPI_BOX = 4096;
constexpr int EPI_WARP_BYTES = 4 * EPI_BOX;
static_assert(CVT_WARPS * EPI_WARP_BYTES <= OFF_SCALE, "epilogue boxes must fit the free rings");

struct Params {
  const float* scale;
  void* y;
  const void* residual;
  int M, N, K;
  int y_fmt;    // FMT_BF16 / FMT_F16 / FMT_F32
  int res_fmt;  // -1 none, FMT_BF16 / FMT_F16 / FMT_F32
  int act;      // 0 none, 1 GELU
  int gelu_tanh;
  int kb_per_split;  // k-blocks per split (grid.z splits, fp32 partial outputs); all of K when not split
};

// GELU, exact form: x * Phi(x), Phi the standard normal CDF.  Phi(-|x|) = erfc(|x| / sqrt 2) / 2
// is evaluated with Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26:
// erfc(z) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2) + e(z), t = 1 / (1 + p z),
// |e(z)| <= 1.5e-7 for z >= 0, here with the hardware reciprocal and base-2 exponential.  Branch-free;
// huge |x| gives x (x >= 0) or 0 (x < 0).
__device__ __forceinline__ float gelu_erf(float x) {
  constexpr float p = 0.3275911f;
  // A&S coefficients, halved so that the sum is Phi(-|x|) rather than erfc
  constexpr float a1 = 0.5f * 0.254829592f, a2 = 0.5f * -0.284496736f, a3 = 0.5f * 1.421413741f,
                  a4 = 0.5f * -1.453152027f, a5 = 0.5f * 1.061405429f;
  const float ax = fabsf(x);
  const float t = rcp_approx(fmaf(p * 0.7071067811865476f, ax, 1.f));  // z = |x| / sqrt 2
  const float q = fmaf(fmaf(fmaf(fmaf(a5, t, a4), t, a3), t, a2), t, a1) * t;
  const float e = ex2_approx(x * (x * -0.7213475204444817f));  // exp(-x^2 / 2) = 2^(-x^2 log2(e) / 2)
  // x Phi(x) = max(x, 0) - |x| Phi(-|x|)
  return fmaf(-ax * e, q, fmaxf(x, 0.f));
}

// GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) = x / (1 + exp(-2y)).
__device__ __forceinline__ float gelu_tanh(float x) {
  const float y = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
  return x * rcp_approx(1.f + ex2_approx(-2.8853900817779268f * y));  // exp(-2y) = 2^(-2y log2(e))
}

template <bool F16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_w8a16_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_r, const Params p,
                      const KernelGuard guard) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem + OFF_X;
  uint8_t* sW8 = smem + OFF_W8;
  uint8_t* sW16 = smem + OFF_W16;
  float* sScale = reinterpret_cast<float*>(smem + OFF_SCALE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* x_full = bars;                      // leader: both CTAs' activation halves landed
  uint64_t* w8_full = x_full + RAW_STAGES;      // this CTA's e4m3 rows landed
  uint64_t* raw_empty = w8_full + RAW_STAGES;   // pair MMAs done with the activations + e4m3 rows read
  uint64_t* w16_full = raw_empty + RAW_STAGES;  // leader: both CTAs' widened rows written
  uint64_t* w16_empty = w16_full + CVT_STAGES;  // pair MMAs done with the widened rows
  uint64_t* acc_full = w16_empty + CVT_STAGES;
  uint64_t* drain_bar = acc_full + 1;
  uint64_t* res_full = drain_bar + 1;  // per epilogue warp, two residual boxes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int tile_m = blockIdx.x >> 1;  // pair tile of 256 tokens
  const int tile_n = blockIdx.y;       // pair tile of 512 channels
  const int tok_cta = tile_m * BM + static_cast<int>(rank) * BM_CTA;  // this CTA's 128 tokens
  const int kb_total = (p.K + BK - 1) / BK;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int num_kb = min(kb_total - kb0, p.kb_per_split);
  // weight rows this CTA widens: block b holds channels tile_n*512 + b*256 + rank*128 + [0, 128)
  auto w_row0 = [&](int b) { return tile_n * BN + b * BN_MMA + static_cast<int>(rank) * 128; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_STAGES; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&w8_full[s], 1);
      mbar_init(&raw_empty[s], 1 + CVT_WARPS);  // MMA commit + this CTA's converter warps
    }
    for (int c = 0; c < CVT_STAGES; ++c) {
      mbar_init(&w16_full[c], 2 * CVT_WARPS);  // used in the leader: both CTAs' converter warps
      mbar_init(&w16_empty[c], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    for (int i = 0; i < 2 * CVT_WARPS; ++i) mbar_init(&res_full[i], 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_y);
    if (p.res_fmt >= 0) tma_prefetch_desc(&tm_r);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  for (int i = threadIdx.x; i < BN; i += THREADS) {
    const int n = tile_n * BN + i;
    sScale[i] = n < p.N ? p.scale[n] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    int issued = 0;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % RAW_STAGES;
      const uint32_t it = static_cast<uint32_t>(kb / RAW_STAGES);
      if (!mbar_wait(&raw_empty[s], (it & 1u) ^ 1u, guard, abort_flag,
                     where_code(ERR_TIMEOUT_GEMM_PRODUCER, rank, kb)))
        break;
      if (lane == 0) {
        const int k = (kb0 + kb) * BK;
        mbar_arrive_expect_tx(&w8_full[s], W8_BYTES);
        tma_load_2d(sW8 + s * W8_BYTES, &tm_w, &w8_full[s], k, w_row0(0));
        tma_load_2d(sW8 + s * W8_BYTES + W8_BLOCK, &tm_w, &w8_full[s], k, w_row0(1));
        if (leader) mbar_arrive_expect_tx(&x_full[s], 2 * X_BYTES);
        tma_load_2d_pair(sX + s * X_BYTES, &tm_x, mapa_shared(smem_u32(&x_full[s]), 0), k, tok_cta);
      }
      __syncwarp();
      issued = kb + 1;
    }
    // Never leave with copies in flight: every CTA drains its weight loads; the leader's
    // activation barrier counts both CTAs' activation loads, and the peer is held by the
    // final cluster barrier until the leader has drained.
    for (int s = 0; s < RAW_STAGES && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / RAW_STAGES) * RAW_STAGES;
      const uint32_t par = static_cast<uint32_t>(last / RAW_STAGES) & 1u;
      mbar_wait(&w8_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, s), true);
      if (leader) mbar_wait(&x_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, s), true);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only)
    if (leader) {
      constexpr uint32_t idesc = idesc_f16kind(BM, BN_MMA, F16, false, false);
      bool ok = true;
      for (int kb = 0; kb < num_kb && ok; ++kb) {
        const int s = kb % RAW_STAGES;
        const int c = kb % CVT_STAGES;
        ok = mbar_wait(&x_full[s], static_cast<uint32_t>(kb / RAW_STAGES) & 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_GEMM_MMA_X, rank, kb)) &&
             mbar_wait(&w16_full[c], static_cast<uint32_t>(kb / CVT_STAGES) & 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_GEMM_MMA, rank, kb));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t x0 = smem_u32(sX + s * X_BYTES);
          const uint32_t w0 = smem_u32(sW16 + c * W16_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(x0 + kk * 32, 16, 1024);
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              const uint64_t bd = smem_desc_sw128(w0 + b * W16_BLOCK + kk * 32, 16, 1024);
              mma_f16kind_ss_pair(tmem + b * BN_MMA, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          mma_commit_pair(&raw_empty[s], 0x3);
          mma_commit_pair(&w16_empty[c], 0x3);
        }
        __syncwarp();
      }
      if (lane == 0) {
        if (ok) mma_commit_pair(acc_full, 0x3);
        mma_commit_pair(drain_bar, 0x3);  // all MMAs retired before either CTA frees TMEM
      }
      __syncwarp();
    }
    mbar_wait(drain_bar, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN_MMA, rank, 0), true);
  } else {
    // ---------------- converters (warps 2..9): thread = one of this CTA's 256 weight rows
    const int ct = threadIdx.x - 64;  // 0..255
    const int b = ct >> 7;            // which MMA's B half
    const int r = ct & 127;           // row within the 128-row block
    bool ok = true;
    for (int kb = 0; kb < num_kb && ok; ++kb) {
      const int s = kb % RAW_STAGES;
      const int c = kb % CVT_STAGES;
      ok = mbar_wait(&w8_full[s], static_cast<uint32_t>(kb / RAW_STAGES) & 1u, guard, abort_flag,
                     where_code(ERR_TIMEOUT_GEMM_CONVERT, rank, kb)) &&
           mbar_wait(&w16_empty[c], (static_cast<uint32_t>(kb / CVT_STAGES) & 1u) ^ 1u, guard, abort_flag,
                     where_code(ERR_TIMEOUT_GEMM_CONVERT, rank, kb));
      if (!ok) break;
      // e4m3 row: 64 bytes, 64-byte swizzle (16-byte chunk j sits at chunk j ^ ((r >> 1) & 3))
      const uint8_t* src = sW8 + s * W8_BYTES + b * W8_BLOCK + r * BK;
      // widened row: 128 bytes, 128-byte swizzle (chunk j sits at chunk j ^ (r & 7))
      uint8_t* dst = sW16 + c * W16_BYTES + b * W16_BLOCK + r * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + ((q ^ ((r >> 1) & 3)) << 4));
        uint4 o0, o1;
        e4m3x4_to_16x4<F16>(v.x, o0.x, o0.y);
        e4m3x4_to_16x4<F16>(v.y, o0.z, o0.w);
        e4m3x4_to_16x4<F16>(v.z, o1.x, o1.y);
        e4m3x4_to_16x4<F16>(v.w, o1.z, o1.w);
        *reinterpret_cast<uint4*>(dst + (((2 * q) ^ (r & 7)) << 4)) = o0;
        *reinterpret_cast<uint4*>(dst + (((2 * q + 1) ^ (r & 7)) << 4)) = o1;
      }
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_remote(mapa_shared(smem_u32(&w16_full[c]), 0));
        mbar_arrive(&raw_empty[s]);
      }
    }

    // ---------------- epilogue: TMEM lane = token, column = channel of accumulator `acc`.
    // Per 32-channel chunk a warp reads its 32 tokens' accumulators, scales (and activates)
    // them, adds the residual box that TMA brought into shared memory, writes the result row
    // by row into a swizzled output box and hands the box to a TMA store.  Global traffic is
    // all asynchronous: the residual boxes of the next two chunks and the stores of the last
    // two are in flight while a chunk is computed.
    if (ok && mbar_wait(acc_full, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_EPILOGUE, rank, 0))) {
      tc_fence_after();
      const int ew = warp - 2;
      const int quarter = warp & 3;
      const int acc = ew >> 2;
      const int tok_warp = tok_cta + quarter * 32;
      const int ch_warp = tile_n * BN + acc * BN_MMA;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN_MMA;
      uint8_t* ebox = smem + OFF_X + ew * EPI_WARP_BYTES;  // out box 0, out box 1, residual 0, residual 1
      uint64_t* rbar = res_full + 2 * ew;
      // valid chunks (N % 32 == 0); none when all 32 of the warp's tokens lie beyond M
      const int nch = tok_warp < p.M ? min(BN_MMA, p.N - ch_warp) / 32 : 0;
      const bool has_res = p.res_fmt >= 0;
      const uint32_t res_box_bytes = p.res_fmt == FMT_F32 ? 4096u : 2048u;
      auto issue_res = [&](int c) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&rbar[c & 1], res_box_bytes);
        tma_load_2d(ebox + (2 + (c & 1)) * EPI_BOX, &tm_r, &rbar[c & 1], ch_warp + 32 * c, tok_warp);
      };
      int res_issued = 0;
      if (has_res && lane == 0) {
        for (; res_issued < min(2, nch); ++res_issued) issue_res(res_issued);
      }
      res_issued = __shfl_sync(0xffffffffu, res_issued, 0);
      int c = 0;
      for (; c < nch; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + 32 * c, r);
        tmem_ld_wait();
        const int col = acc * BN_MMA + 32 * c;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) * sScale[col + j];
        if (p.act == 1) {
          if (p.gelu_tanh) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_erf(v[j]);
          }
        }
        if (has_res) {
          if (!mbar_wait(&rbar[c & 1], static_cast<uint32_t>(c >> 1) & 1u, guard, abort_flag,
                         where_code(ERR_TIMEOUT_GEMM_EPILOGUE, rank, 1 + c)))
            break;
          const uint8_t* rrow = ebox + (2 + (c & 1)) * EPI_BOX;
          if (p.res_fmt == FMT_F32) {  // 128-byte rows, 128-byte swizzle
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 t = *reinterpret_cast<const float4*>(rrow + lane * 128 + ((q ^ (lane & 7)) << 4));
              v[4 * q] += t.x; v[4 * q + 1] += t.y; v[4 * q + 2] += t.z; v[4 * q + 3] += t.w;
            }
          } else {  // 64-byte rows, 64-byte swizzle
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 t = *reinterpret_cast<const uint4*>(rrow + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4));
              const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                v[8 * q + 2 * k] += p.res_fmt == FMT_F16 ? f16_lo(w[k]) : bf16_lo(w[k]);
                v[8 * q + 2 * k + 1] += p.res_fmt == FMT_F16 ? f16_hi(w[k]) : bf16_hi(w[k]);
              }
            }
          }
        }
        // output box c & 1: the store issued two chunks ago must have read it
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* orow = ebox + (c & 1) * EPI_BOX;
        if (p.y_fmt == FMT_F32) {  // 128-byte rows, 128-byte swizzle
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(orow + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {  // 64-byte rows, 64-byte swizzle
          const bool f16 = p.y_fmt == FMT_F16;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = f16 ? pack_f16x2(v[8 * q], v[8 * q + 1]) : pack_bf16x2(v[8 * q], v[8 * q + 1]);
            o.y = f16 ? pack_f16x2(v[8 * q + 2], v[8 * q + 3]) : pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
            o.z = f16 ? pack_f16x2(v[8 * q + 4], v[8 * q + 5]) : pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
            o.w = f16 ? pack_f16x2(v[8 * q + 6], v[8 * q + 7]) : pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
            *reinterpret_cast<uint4*>(orow + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) = o;
          }
        }
        fence_proxy_async_smem();  // generic writes -> visible to the TMA store
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_y, orow, ch_warp + 32 * c, tok_warp, blockIdx.z);  // rows >= M are clipped
          bulk_commit_group();
          if (has_res && res_issued < nch) issue_res(res_issued);  // into the residual box just read
        }
        if (has_res && res_issued < nch) ++res_issued;
      }
      // nothing in flight when the CTA moves on: residual loads not consumed, stores' reads
      if (lane == 0) {
        for (int k = c; k < res_issued; ++k)
          mbar_wait(&rbar[k & 1], static_cast<uint32_t>(k >> 1) & 1u, guard, abort_flag,
                    where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, 0x100 + k), true);
        bulk_wait_group_read<0>();
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair MMAs or remote arrives may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// out[i] = sum over splits of part[z][i], as bf16; 8 elements per thread.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, uint16_t* __restrict__ out, int64_t n,
                                     int splits) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= n / 8) return;
  float v[8];
  load8<FMT_F32>(part, i, v);
  for (int z = 1; z < splits; ++z) {
    float w[8];
    load8<FMT_F32>(part + z * n, i, w);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] += w[k];
  }
  store8<FMT_BF16>(out, i, v);
}

}  // namespace gemm

int gemm_pick_splits(int M, int N, int K) {
  // The split count whose tile grid fills the pairs of SMs best (ties: fewer splits).
  const int tiles = ((M + gemm::BM - 1) / gemm::BM) * ((N + gemm::BN - 1) / gemm::BN);
  const int kb = (K + gemm::BK - 1) / gemm::BK;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 8 && s <= kb / 16; ++s) {
    const int t = tiles * s;
    const int waves = (t + gemm::MAX_PAIRS - 1) / gemm::MAX_PAIRS;
    const double eff = static_cast<double>(t) / (static_cast<double>(waves) * gemm::MAX_PAIRS);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_splitk_reduce(const float* part, uint16_t* out, int64_t n, int splits, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  gemm::splitk_reduce_kernel<<<static_cast<unsigned>((n / 8 + 255) / 256), 256, 0, s>>>(part, out, n, splits);
  return cudaGetLastError();
}

cudaError_t launch_gemm_w8a16(const GemmArgs& a, const KernelGuard& g, cudaStream_t s) {
  using namespace gemm;
  if (a.M <= 0 || a.N <= 0) return cudaSuccess;
  const bool f16 = a.a_fmt == FMT_F16;
  CUtensorMap tm_x, tm_w;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K)};
    const uint32_t box[2] = {BK, 128};
    if (!make_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.w), dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K) * 2};
    const uint32_t box[2] = {BK, BM_CTA};  // each CTA of the pair loads its own 128 rows
    if (!make_tmap(&tm_x, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(a.a), dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const int kb_total = (a.K + BK - 1) / BK;
  const int splits_req = a.k_splits > 1 ? a.k_splits : 1;
  const int kb_per = (kb_total + splits_req - 1) / splits_req;
  const int splits = (kb_total + kb_per - 1) / kb_per;
  if (splits > 1 && (a.y_fmt != FMT_F32 || a.residual != nullptr || a.act != 0)) return cudaErrorInvalidValue;
  // output: [splits][M][N] (one fp32 partial per split when K is split), 32 x 32 boxes
  CUtensorMap tm_y, tm_r;
  auto tdt = [](int fmt) {
    return fmt == FMT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                          : (fmt == FMT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  };
  auto tswz = [](int fmt) { return fmt == FMT_F32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B; };
  {
    const uint64_t esz = a.y_fmt == FMT_F32 ? 4 : 2;
    const uint64_t dims[3] = {static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M), static_cast<uint64_t>(splits)};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.N) * esz, static_cast<uint64_t>(a.N) * a.M * esz};
    const uint32_t box[3] = {32, 32, 1};
    if (!make_tmap(&tm_y, tdt(a.y_fmt), 3, a.y, dims, strides, box, tswz(a.y_fmt))) return cudaErrorInvalidValue;
  }
  memset(&tm_r, 0, sizeof(tm_r));
  if (a.residual != nullptr) {
    const uint64_t esz = a.res_fmt == FMT_F32 ? 4 : 2;
    const uint64_t dims[2] = {static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.N) * esz};
    const uint32_t box[2] = {32, 32};
    if (!make_tmap(&tm_r, tdt(a.res_fmt), 2, const_cast<void*>(a.residual), dims, strides, box, tswz(a.res_fmt)))
      return cudaErrorInvalidValue;
  }
  Params p{a.scale, a.y, a.residual, a.M, a.N, a.K, a.y_fmt, a.residual ? a.res_fmt : -1, a.act, a.gelu_tanh, kb_per};
  dim3 grid(2 * ((a.M + BM - 1) / BM), (a.N + BN - 1) / BN, splits);
  auto kern = f16 ? gemm_w8a16_kernel<true> : gemm_w8a16_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, THREADS, SMEM_BYTES, s>>>(tm_x, tm_w, tm_y, tm_r, p, g);
  return cudaGetLastError();
}

}  // namespace jab
