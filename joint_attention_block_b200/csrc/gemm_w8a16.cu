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
// The kernel is persistent: one pair of CTAs per pair of SMs walks the work units
// (tile_m, tile_n, K split) pair_id, pair_id + pairs, ...  The rings run on across
// units, so the producer loads the next unit's first stages while the current
// unit's epilogue runs, and no CTA is relaunched per tile.
//
// Per CTA:
//   warp 0      TMA producer: 128 x 64 activations (128B swizzle) and 2 x (128 x 64
//               bytes) e4m3 weights (64B swizzle) per stage, 3-stage ring.
//   warp 1      TMEM allocation (pair); in the leader, one lane issues 2 x 4 pair
//               MMAs per stage.
//   warps 2..9  converters: thread = one weight row; widen 64 e4m3 bytes to f16 (or
//               bf16) and store them into the 2-stage widened ring.  After a unit's
//               last stage, the epilogue: thread = one token row of TMEM (warp w reads
//               lanes 32*(w%4).., accumulator (w-2)/4), scale, optional GELU, optional
//               residual (TMA-loaded boxes), 32 x 32 output boxes stored by TMA.  The
//               output boxes live in the widened ring (idle until these same warps
//               convert the next unit); the channel scales and the first residual
//               boxes live past it and are fetched while the unit's last MMAs run.
//               The next unit's MMAs wait for both CTAs' converters, hence for both
//               epilogues to have read TMEM.
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
// For weights larger than L2 (the 218 MB conditioning projection, read once from DRAM), the producer
// also asks L2 for the tiles PREFETCH_KB stages ahead of the ring (~5 us of MMAs), so that the
// ring's own loads find them there.  Measured: the conditioning projection 2 % faster; the
// L2-resident block GEMMs lose about 1 % with it, so they run without.
constexpr int PREFETCH_KB = 4;
constexpr int64_t PREFETCH_MIN_W8_BYTES = 100ll << 20;

constexpr int OFF_X = 0;
constexpr int OFF_W8 = OFF_X + RAW_STAGES * X_BYTES;
constexpr int OFF_W16 = OFF_W8 + RAW_STAGES * W8_BYTES;
// Epilogue boxes of 32 tokens x 32 channels (2 KB in 16-bit, 4 KB in fp32).  Per epilogue
// warp: 8 KB over the widened ring for its two output boxes (one when both the output and
// the residual are fp32) and, with an fp32 residual, its second residual box; 4 KB past the
// ring for the first residual box(es) (both 16-bit boxes, or the first fp32 box), which can
// therefore be loaded while the unit's last MMAs still read the ring.
constexpr int EPI_RING_WARP = 8 * 1024;
constexpr int EPI_EXTRA_WARP = 4 * 1024;
constexpr int OFF_EPI = OFF_W16;
constexpr int OFF_EPI_EXTRA = OFF_W16 + CVT_STAGES * W16_BYTES;
constexpr int OFF_SCALE = OFF_EPI_EXTRA + CVT_WARPS * EPI_EXTRA_WARP;  // per epilogue warp, 256 scales
static_assert(CVT_WARPS * EPI_RING_WARP <= CVT_STAGES * W16_BYTES, "output boxes fit over the widened ring");
constexpr int OFF_BAR = OFF_SCALE + CVT_WARPS * BN_MMA * 4;
constexpr int NUM_BARS = 3 * RAW_STAGES + 2 * CVT_STAGES + 3 + 2 * CVT_WARPS;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

struct Params {
  const float* scale;
  void* y;
  const void* residual;
  int M, N, K;
  int y_fmt;    // FMT_BF16 / FMT_F16 / FMT_F32
  int res_fmt;  // -1 none, FMT_BF16 / FMT_F16 / FMT_F32
  int act;      // 0 none, 1 GELU
  int gelu_tanh;
  int kb_per_split;  // k-blocks per split (fp32 partial outputs per split); all of K when not split
  int tiles_m, tiles_n, units;  // work units: tile_m fastest, then tile_n, then the K split
  int y_evict_first;            // output stream larger than L2: store it with an evict-first hint
  int prefetch;                 // weight larger than L2: prefetch the tiles ahead into L2
};

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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* x_full = bars;                      // leader: both CTAs' activation halves landed
  uint64_t* w8_full = x_full + RAW_STAGES;      // this CTA's e4m3 rows landed
  uint64_t* raw_empty = w8_full + RAW_STAGES;   // pair MMAs done with the activations + e4m3 rows read
  uint64_t* w16_full = raw_empty + RAW_STAGES;  // leader: both CTAs' widened rows written
  uint64_t* w16_empty = w16_full + CVT_STAGES;  // pair MMAs done with the widened rows
  uint64_t* acc_full = w16_empty + CVT_STAGES;  // one phase per unit
  uint64_t* drain_bar = acc_full + 1;
  uint64_t* epi_done = drain_bar + 1;  // all epilogue warps of this CTA are done with a unit
  uint64_t* res_full = epi_done + 1;   // per epilogue warp, two residual boxes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;
  const int kb_total = (p.K + BK - 1) / BK;
  struct Unit {
    int tile_m, tile_n, split, tok_cta, kb0, num_kb;
  };
  auto unit = [&](int u) {
    Unit w;
    w.tile_m = u % p.tiles_m;
    w.tile_n = (u / p.tiles_m) % p.tiles_n;
    w.split = u / (p.tiles_m * p.tiles_n);
    w.tok_cta = w.tile_m * BM + static_cast<int>(rank) * BM_CTA;  // this CTA's 128 tokens
    w.kb0 = w.split * p.kb_per_split;
    w.num_kb = min(kb_total - w.kb0, p.kb_per_split);
    return w;
  };

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
    mbar_init(epi_done, CVT_WARPS);
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
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_then_release();  // the setup above overlaps the previous kernel's tail

  if (warp == 0) {
    // ---------------- TMA producer: runs ahead across units, bounded by the raw ring
    int g = 0;  // stages issued so far (all units)
    bool ok = true;
    for (int u = pair; u < p.units && ok; u += pairs) {
      const Unit w = unit(u);
      for (int kb = 0; kb < w.num_kb; ++kb) {
        const int s = g % RAW_STAGES;
        const uint32_t it = static_cast<uint32_t>(g / RAW_STAGES);
        if (!mbar_wait(&raw_empty[s], (it & 1u) ^ 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_GEMM_PRODUCER, rank, g))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const int k = (w.kb0 + kb) * BK;
          const int wr = w.tile_n * BN + static_cast<int>(rank) * 128;  // block b adds b * 256
          mbar_arrive_expect_tx(&w8_full[s], W8_BYTES);
          tma_load_2d(sW8 + s * W8_BYTES, &tm_w, &w8_full[s], k, wr);
          tma_load_2d(sW8 + s * W8_BYTES + W8_BLOCK, &tm_w, &w8_full[s], k, wr + BN_MMA);
          if (leader) mbar_arrive_expect_tx(&x_full[s], 2 * X_BYTES);
          tma_load_2d_pair(sX + s * X_BYTES, &tm_x, mapa_shared(smem_u32(&x_full[s]), 0), k, w.tok_cta);
          if (p.prefetch && kb + PREFETCH_KB < w.num_kb) {  // this unit's tiles PREFETCH_KB stages ahead
            const int kp = k + PREFETCH_KB * BK;
            tma_prefetch_l2_2d(&tm_w, kp, wr);
            tma_prefetch_l2_2d(&tm_w, kp, wr + BN_MMA);
            tma_prefetch_l2_2d(&tm_x, kp, w.tok_cta);
          }
        }
        __syncwarp();
        ++g;
      }
    }
    // Never leave with copies in flight: every CTA drains its weight loads; the leader's
    // activation barrier counts both CTAs' activation loads, and the peer is held by the
    // final cluster barrier until the leader has drained.
    for (int s = 0; s < RAW_STAGES && s < g; ++s) {
      const int last = s + ((g - 1 - s) / RAW_STAGES) * RAW_STAGES;
      const uint32_t par = static_cast<uint32_t>(last / RAW_STAGES) & 1u;
      mbar_wait(&w8_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, s), true);
      if (leader) mbar_wait(&x_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, s), true);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only)
    if (leader) {
      constexpr uint32_t idesc = idesc_f16kind(BM, BN_MMA, F16, false, false);
      bool ok = true;
      int g = 0;
      for (int u = pair; u < p.units && ok; u += pairs) {
        const Unit w = unit(u);
        for (int kb = 0; kb < w.num_kb; ++kb) {
          const int s = g % RAW_STAGES;
          const int c = g % CVT_STAGES;
          // the first stage of a unit also waits, through the converters, for both epilogues
          // of the previous unit to have read the accumulators
          ok = mbar_wait(&x_full[s], static_cast<uint32_t>(g / RAW_STAGES) & 1u, guard, abort_flag,
                         where_code(ERR_TIMEOUT_GEMM_MMA_X, rank, g)) &&
               mbar_wait(&w16_full[c], static_cast<uint32_t>(g / CVT_STAGES) & 1u, guard, abort_flag,
                         where_code(ERR_TIMEOUT_GEMM_MMA, rank, g));
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
            if (kb + 1 == w.num_kb) mma_commit_pair(acc_full, 0x3);  // this unit's accumulators
          }
          __syncwarp();
          ++g;
        }
      }
      if (lane == 0) mma_commit_pair(drain_bar, 0x3);  // all MMAs retired before either CTA frees TMEM
      __syncwarp();
    }
    mbar_wait(drain_bar, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN_MMA, rank, 0), true);
  } else {
    // ---------------- converters + epilogue (warps 2..9)
    const int ct = threadIdx.x - 64;  // converter: one of this CTA's 256 weight rows
    const int b = ct >> 7;            // which MMA's B half
    const int r = ct & 127;           // row within the 128-row block
    const int ew = warp - 2;          // epilogue: warp index
    const int quarter = warp & 3;
    const int acc = ew >> 2;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN_MMA;
    float* sScale = reinterpret_cast<float*>(smem + OFF_SCALE) + ew * BN_MMA;
    const bool has_res = p.res_fmt >= 0;
    const bool res32 = p.res_fmt == FMT_F32;
    const int out_box = 32 * 32 * (p.y_fmt == FMT_F32 ? 4 : 2);
    const int res_box = has_res ? 32 * 32 * (res32 ? 4 : 2) : 0;
    // two output boxes, except fp32 out with an fp32 residual (whose second box shares the
    // warp's ring part), which gets one
    const int n_out = 2 * out_box + (res32 ? res_box : 0) <= EPI_RING_WARP ? 2 : 1;
    uint8_t* const ebox = smem + OFF_EPI + ew * EPI_RING_WARP;  // output boxes [, fp32 residual box 1]
    uint8_t* const rbox0 = smem + OFF_EPI_EXTRA + ew * EPI_EXTRA_WARP;
    uint8_t* const rbox1 = res32 ? ebox + n_out * out_box : rbox0 + res_box;
    const int n_early = res32 ? 1 : 2;  // residual boxes past the ring
    uint64_t* rbar = res_full + 2 * ew;
    uint32_t rph = 0u;  // bit b: phase parity of residual box b
    bool ok = true;
    int g = 0;
    int ui = 0;
    for (int u = pair; u < p.units && ok; u += pairs, ++ui) {
      const Unit w = unit(u);
      // the epilogue boxes overlap the widened ring: no warp converts for this unit until
      // every warp has finished the previous unit's epilogue
      if (ui > 0 && !mbar_wait(epi_done, static_cast<uint32_t>(ui - 1) & 1u, guard, abort_flag,
                               where_code(ERR_TIMEOUT_GEMM_CONVERT, rank, 0xFFFF))) {
        ok = false;
        break;
      }
      for (int kb = 0; kb < w.num_kb; ++kb) {
        const int s = g % RAW_STAGES;
        const int c = g % CVT_STAGES;
        ok = mbar_wait(&w8_full[s], static_cast<uint32_t>(g / RAW_STAGES) & 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_GEMM_CONVERT, rank, g)) &&
             mbar_wait(&w16_empty[c], (static_cast<uint32_t>(g / CVT_STAGES) & 1u) ^ 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_GEMM_CONVERT, rank, g));
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
        tc_fence_before();         // and the previous unit's TMEM reads ordered before its MMAs
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_remote(mapa_shared(smem_u32(&w16_full[c]), 0));
          mbar_arrive(&raw_empty[s]);
        }
        ++g;
      }
      if (!ok) break;

      // ---------------- epilogue of unit u: TMEM lane = token, column = channel of `acc`.
      // Per 32-channel chunk a warp reads its 32 tokens' accumulators, scales (and
      // activates) them, adds the residual box that TMA brought into shared memory,
      // writes the result row by row into a swizzled output box and hands the box to a
      // TMA store.  The residual boxes of the next two chunks and the stores of the last
      // two are in flight while a chunk is computed.
      const int tok_warp = w.tok_cta + quarter * 32;
      const int ch_warp = w.tile_n * BN + acc * BN_MMA;
      // valid chunks (N % 32 == 0); none when all 32 of the warp's tokens lie beyond M
      const int nch = tok_warp < p.M ? min(BN_MMA, p.N - ch_warp) / 32 : 0;
      {  // this warp's 256 channel scales, loaded while the unit's last MMAs run
        const int n0 = ch_warp + 8 * lane;
#pragma unroll
        for (int k = 0; k < 8; ++k) sScale[8 * lane + k] = n0 + k < p.N ? p.scale[n0 + k] : 0.f;
      }
      auto issue_res = [&](int c) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&rbar[c & 1], static_cast<uint32_t>(res_box));
        tma_load_2d((c & 1) ? rbox1 : rbox0, &tm_r, &rbar[c & 1], ch_warp + 32 * c, tok_warp);
      };
      // the residual boxes past the ring are loaded while the unit's last MMAs run
      int res_issued = 0;
      if (has_res && lane == 0) {
        for (; res_issued < min(n_early, nch); ++res_issued) issue_res(res_issued);
      }
      if (!mbar_wait(acc_full, static_cast<uint32_t>(ui) & 1u, guard, abort_flag,
                     where_code(ERR_TIMEOUT_GEMM_EPILOGUE, rank, ui))) {
        ok = false;
        if (lane == 0) {  // no residual load left in flight
          for (int k = 0; k < res_issued; ++k) {
            mbar_wait(&rbar[k & 1], (rph >> (k & 1)) & 1u, guard, abort_flag,
                      where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, 0x200 + k), true);
            rph ^= 1u << (k & 1);
          }
        }
        __syncwarp();
        break;
      }
      tc_fence_after();
      __syncwarp();
      if (has_res && lane == 0) {
        for (; res_issued < min(2, nch); ++res_issued) issue_res(res_issued);
      }
      res_issued = __shfl_sync(0xffffffffu, res_issued, 0);
      int c = 0;
      for (; c < nch; ++c) {
        uint32_t rr[32];
        tmem_ld32(taddr + 32 * c, rr);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(rr[j]) * sScale[32 * c + j];
        if (p.act == 1) {
          if (p.gelu_tanh) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 g = gelu_erf_pair(make_float2(v[j], v[j + 1]));
              v[j] = g.x;
              v[j + 1] = g.y;
            }
          }
        }
        if (has_res) {
          const int bx = c & 1;
          if (!mbar_wait(&rbar[bx], (rph >> bx) & 1u, guard, abort_flag,
                         where_code(ERR_TIMEOUT_GEMM_EPILOGUE, rank, 0x100 + c))) {
            ok = false;
            break;
          }
          rph ^= 1u << bx;
          const uint8_t* rrow = bx ? rbox1 : rbox0;
          if (res32) {  // 128-byte rows, 128-byte swizzle
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 t = *reinterpret_cast<const float4*>(rrow + lane * 128 + ((q ^ (lane & 7)) << 4));
              v[4 * q] += t.x; v[4 * q + 1] += t.y; v[4 * q + 2] += t.z; v[4 * q + 3] += t.w;
            }
          } else {  // 64-byte rows, 64-byte swizzle
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 t = *reinterpret_cast<const uint4*>(rrow + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4));
              const uint32_t wv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                v[8 * q + 2 * k] += p.res_fmt == FMT_F16 ? f16_lo(wv[k]) : bf16_lo(wv[k]);
                v[8 * q + 2 * k + 1] += p.res_fmt == FMT_F16 ? f16_hi(wv[k]) : bf16_hi(wv[k]);
              }
            }
          }
        }
        // output box c % n_out: the store issued n_out chunks ago must have read it
        if (lane == 0) {
          if (n_out == 2) bulk_wait_group_read<1>();
          else bulk_wait_group_read<0>();
        }
        __syncwarp();
        uint8_t* orow = ebox + (c % n_out) * out_box;
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
          if (p.y_evict_first)  // keep the re-read activation tiles in L2, not the output
            tma_store_3d_hint(&tm_y, orow, ch_warp + 32 * c, tok_warp, w.split, l2_evict_first_policy());
          else
            tma_store_3d(&tm_y, orow, ch_warp + 32 * c, tok_warp, w.split);  // rows >= M are clipped
          bulk_commit_group();
          if (has_res && res_issued < nch) issue_res(res_issued);  // into the residual box just read
        }
        if (has_res && res_issued < nch) ++res_issued;
      }
      // Nothing in flight past the unit: residual loads not consumed (after a failed wait),
      // and the stores' reads of the boxes, which the next unit's conversions overwrite.
      if (lane == 0) {
        for (int k = c; k < res_issued; ++k) {
          mbar_wait(&rbar[k & 1], (rph >> (k & 1)) & 1u, guard, abort_flag,
                    where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, 0x200 + k), true);
          rph ^= 1u << (k & 1);
        }
        bulk_wait_group_read<0>();
      }
      rph = __shfl_sync(0xffffffffu, rph, 0);
      __syncwarp();
      if (!ok) break;
      if (lane == 0) mbar_arrive(epi_done);
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
  pdl_wait_then_release();
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
  // The fewest K splits whose tile grid fills the pairs of SMs within 2 % of the best split count
  // up to 16 (each split adds an fp32 partial of the output to write and reduce).
  const int tiles = ((M + gemm::BM - 1) / gemm::BM) * ((N + gemm::BN - 1) / gemm::BN);
  const int kb = (K + gemm::BK - 1) / gemm::BK;
  double eff[17] = {0.0};
  double best_eff = 0.0;
  for (int s = 1; s <= 16 && s <= kb / 16; ++s) {
    const int t = tiles * s;
    const int waves = (t + gemm::MAX_PAIRS - 1) / gemm::MAX_PAIRS;
    eff[s] = static_cast<double>(t) / (static_cast<double>(waves) * gemm::MAX_PAIRS);
    if (eff[s] > best_eff) best_eff = eff[s];
  }
  for (int s = 1; s <= 16 && s <= kb / 16; ++s)
    if (eff[s] >= best_eff - 0.02) return s;
  return 1;
}

cudaError_t launch_splitk_reduce(const float* part, uint16_t* out, int64_t n, int splits, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  launch_pdl(gemm::splitk_reduce_kernel, dim3(static_cast<unsigned>((n / 8 + 255) / 256)), dim3(256), 0, s, part, out, n,
             splits);
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
  const int tiles_m = (a.M + BM - 1) / BM, tiles_n = (a.N + BN - 1) / BN;
  const int units = tiles_m * tiles_n * splits;
  // outputs of more than ~100 MB (the QKV and MLP-up projections at 1024 px) cannot stay in the
  // 126 MB L2 anyway; smaller ones (O's fp32 residual stream) are read back from L2 by the next kernel
  const int64_t y_bytes = static_cast<int64_t>(a.M) * a.N * (a.y_fmt == FMT_F32 ? 4 : 2) * splits;
  Params p{a.scale, a.y,  a.residual, a.M,   a.N,     a.K,     a.y_fmt, a.residual ? a.res_fmt : -1,
           a.act,   a.gelu_tanh, kb_per, tiles_m, tiles_n, units, y_bytes > (100ll << 20) ? 1 : 0,
           static_cast<int64_t>(a.N) * a.K >= PREFETCH_MIN_W8_BYTES ? 1 : 0};
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 2 * MAX_PAIRS;
  const int pairs = min(units, max(1, sms / 2));
  dim3 grid(2 * pairs, 1, 1);
  auto kern = f16 ? gemm_w8a16_kernel<true> : gemm_w8a16_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, grid, dim3(THREADS), SMEM_BYTES, s, tm_x, tm_w, tm_y, tm_r, p, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace jab
