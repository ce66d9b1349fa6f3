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
// The kernel computes the transposed tile D = W8_tile * A_tile^T so that the
// widened weights are the MMA's A operand and live in TENSOR MEMORY: TMA brings
// each CTA's e4m3 weight tile (128 rows x 64 bytes) into shared memory, each
// converter thread owns one weight row (one TMEM lane), widens its bytes in
// registers and writes them with tcgen05.st.  The 16-bit weights never touch
// shared memory.
//
// Two CTAs on two SMs (a cluster of 2) share one 256 (channels) x 256 (tokens) tile
// through the pair form of the MMA (tcgen05.mma.cta_group::2, M = 256, N = 256):
// each CTA widens its own 128 weight rows into its own TMEM (half of A) and
// TMA-loads its own 128 tokens into its own shared memory (half of B); the leader
// CTA issues the MMAs, each CTA's TMEM receives its 128 channels x 256 tokens of D.
// Per SM and K-step this reads half the activation bytes of a one-SM 128 x 256
// tile, which is what keeps L2 traffic per FLOP low enough for the tensor pipe.
// Both CTAs' TMA loads count on the leader's barrier, both CTAs' converter warps
// arrive on the leader's barrier, and the leader's MMA commits arrive on both CTAs'
// barriers.  No TMA load is multicast.
//
// Per CTA: 128 channels x 256 tokens x 64 (K) per stage; grid.z = K splits.
//   warp 0      TMA producer: this CTA's 128 x 64 activation half (128B swizzle) and
//               its 128 x 64-byte e4m3 weight tile (64B swizzle), 6-stage rings.
//   warp 1      TMEM allocation (pair); in the leader, one lane issues the pair MMAs.
//   warps 2..9  converters: warp w owns TMEM lanes 32*(w%4).. (channels) and half of
//               each stage's 64 K-columns (TMEM ring of widened weights).  Then the
//               epilogue: tcgen05.ld of the accumulator (lane = channel, column =
//               token), scale, optional GELU, a transpose through shared memory,
//               optional residual, and row-contiguous stores.
#include "common.cuh"

namespace jab {
namespace gemm {

constexpr int BM = 256;      // tokens per pair tile (MMA N)
constexpr int BM_CTA = 128;  // tokens each CTA loads
constexpr int BN = 256;      // output channels per pair tile (MMA M)
constexpr int BN_CTA = 128;  // channels each CTA owns (its TMEM lanes)
constexpr int BK = 64;
constexpr int STAGES = 6;    // activation (smem) and widened-weight (TMEM) ring depth
constexpr int X_BYTES = BM_CTA * BK * 2;  // one TMA box of {BK, BM_CTA} 16-bit elements
constexpr int W_BYTES = BN_CTA * BK;      // one TMA box of {BK, BN_CTA} e4m3 bytes (64-byte swizzle)
constexpr int THREADS = 320;
constexpr int CVT_WARPS = 8;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;   // accumulator: columns [0, 256)
constexpr int A_COL = 256;   // widened weights: stage s at 256 + 32 * s
constexpr int EPI_BYTES = 32 * 32 * 4;  // per-warp transpose buffer

constexpr int OFF_X = 0;
constexpr int OFF_W = OFF_X + STAGES * X_BYTES;
constexpr int OFF_EPI = OFF_W + STAGES * W_BYTES;
constexpr int OFF_SCALE = OFF_EPI + CVT_WARPS * EPI_BYTES;
constexpr int OFF_BAR = OFF_SCALE + BN_CTA * 4;
constexpr int NUM_BARS = 5 * STAGES + 2;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment

struct Params {
  const float* scale;
  void* y;
  const void* residual;
  int M, N, K;
  int y_fmt;    // FMT_BF16 / FMT_F16 / FMT_F32
  int res_fmt;  // -1 none, FMT_BF16 / FMT_F16 / FMT_F32
  int act;      // 0 none, 1 GELU
  int gelu_tanh;
  int kb_per_split;        // k-blocks per split (grid.z splits); all of K when not split
  int64_t y_split_stride;  // elements between the fp32 partial outputs of consecutive splits
};

__device__ __forceinline__ float gelu_f(float x, int tanh_form) {
  if (tanh_form) {
    const float k0 = 0.7978845608028654f, k1 = 0.044715f;
    return 0.5f * x * (1.f + tanhf(k0 * (x + k1 * x * x * x)));
  }
  return 0.5f * x * (1.f + erff(x * 0.7071067811865476f));
}

template <bool F16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_w8a16_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, const Params p,
                      const KernelGuard guard) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem + OFF_X;
  uint8_t* sW = smem + OFF_W;
  float* sScale = reinterpret_cast<float*>(smem + OFF_SCALE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* x_full = bars;               // leader: both CTAs' activation halves landed
  uint64_t* x_empty = bars + STAGES;     // both: the pair MMAs of the stage are done
  uint64_t* a_full = bars + 2 * STAGES;  // leader: both CTAs' weights widened into TMEM
  uint64_t* a_empty = bars + 3 * STAGES;
  uint64_t* w_full = bars + 4 * STAGES;  // this CTA's e4m3 weight tile landed
  uint64_t* acc_full = bars + 5 * STAGES;
  uint64_t* drain_bar = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int tile_m = blockIdx.x >> 1;  // pair tile of 256 tokens
  const int tile_n = blockIdx.y;       // pair tile of 256 channels
  const int tok_cta = tile_m * BM + static_cast<int>(rank) * BM_CTA;  // rows of A this CTA loads
  const int ch_cta = tile_n * BN + static_cast<int>(rank) * BN_CTA;   // channels this CTA owns
  const int kb_total = (p.K + BK - 1) / BK;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int num_kb = min(kb_total - kb0, p.kb_per_split);
  void* const y_out = static_cast<char*>(p.y) + blockIdx.z * p.y_split_stride * 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
      mbar_init(&a_full[s], 2 * CVT_WARPS);  // used in the leader: both CTAs' converter warps
      mbar_init(&a_empty[s], 1);
      mbar_init(&w_full[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  for (int i = threadIdx.x; i < BN_CTA; i += THREADS) {
    const int n = ch_cta + i;
    sScale[i] = n < p.N ? p.scale[n] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer: this CTA's activation half, counted on the leader's barrier
    int issued = 0;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t it = static_cast<uint32_t>(kb / STAGES);
      if (!mbar_wait(&x_empty[s], (it & 1u) ^ 1u, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_PRODUCER, rank, kb))) break;
      if (lane == 0) {
        // The stage is free once its pair MMAs are done; by then this CTA's converters
        // have also consumed the weight bytes of the stage.
        mbar_arrive_expect_tx(&w_full[s], W_BYTES);
        tma_load_2d(sW + s * W_BYTES, &tm_w, &w_full[s], (kb0 + kb) * BK, ch_cta);
        if (leader) mbar_arrive_expect_tx(&x_full[s], 2 * X_BYTES);
        tma_load_2d_pair(sX + s * X_BYTES, &tm_x, mapa_shared(smem_u32(&x_full[s]), 0), (kb0 + kb) * BK, tok_cta);
      }
      __syncwarp();
      issued = kb + 1;
    }
    // Never leave with copies in flight: every CTA drains its weight loads; the leader's
    // activation barrier counts both CTAs' activation loads, and the peer is held by the
    // final cluster barrier until the leader has drained.
    for (int s = 0; s < STAGES && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / STAGES) * STAGES;
      const uint32_t par = static_cast<uint32_t>(last / STAGES) & 1u;
      mbar_wait(&w_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, s), true);
      if (leader) mbar_wait(&x_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, s), true);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only)
    if (leader) {
      constexpr uint32_t idesc = idesc_f16kind(BN, BM, F16, false, false);
      bool ok = true;
      for (int kb = 0; kb < num_kb && ok; ++kb) {
        const int s = kb % STAGES;
        const uint32_t par = static_cast<uint32_t>(kb / STAGES) & 1u;
        ok = mbar_wait(&x_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_MMA_X, rank, kb)) &&
             mbar_wait(&a_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_MMA, rank, kb));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t x0 = smem_u32(sX + s * X_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(x0 + kk * 32, 16, 1024);
            mma_f16kind_ts_pair(tmem + ACC_COL, tmem + A_COL + 32 * s + 8 * kk, bd, idesc,
                                (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit_pair(&x_empty[s], 0x3);
          mma_commit_pair(&a_empty[s], 0x3);
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
    // ---------------- converters (warps 2..9): thread = weight row, half a stage of K each
    const int quarter = warp & 3;
    const int kh = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;  // TMEM lane = channel within this CTA's half
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t par = static_cast<uint32_t>(kb / STAGES) & 1u;
      if (!mbar_wait(&w_full[s], par, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_CONVERT, rank, kb))) {
        ok = false;
        break;
      }
      // 64-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ ((r >> 1) & 3).
      const uint8_t* wrow = sW + s * W_BYTES + row * BK;
      const uint4 c0 = *reinterpret_cast<const uint4*>(wrow + (((2 * kh) ^ ((row >> 1) & 3)) << 4));
      const uint4 c1 = *reinterpret_cast<const uint4*>(wrow + (((2 * kh + 1) ^ ((row >> 1) & 3)) << 4));
      uint32_t h[16];
      e4m3x4_to_16x4<F16>(c0.x, h[0], h[1]);
      e4m3x4_to_16x4<F16>(c0.y, h[2], h[3]);
      e4m3x4_to_16x4<F16>(c0.z, h[4], h[5]);
      e4m3x4_to_16x4<F16>(c0.w, h[6], h[7]);
      e4m3x4_to_16x4<F16>(c1.x, h[8], h[9]);
      e4m3x4_to_16x4<F16>(c1.y, h[10], h[11]);
      e4m3x4_to_16x4<F16>(c1.z, h[12], h[13]);
      e4m3x4_to_16x4<F16>(c1.w, h[14], h[15]);
      if (!mbar_wait(&a_empty[s], par ^ 1u, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_CONVERT, rank, kb))) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st16(tmem + lane_off + A_COL + 32 * s + 16 * kh, h);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&a_full[s]), 0));
    }

    // ---------------- epilogue: lane = channel, TMEM column = token of the pair tile
    if (ok && mbar_wait(acc_full, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_EPILOGUE, rank, 0))) {
      tc_fence_after();
      float* buf = reinterpret_cast<float*>(smem + OFF_EPI + (warp - 2) * EPI_BYTES);
      const float sc = sScale[row];
      const int ch0 = ch_cta + quarter * 32;  // first channel of this warp
      const bool warp_has_channels = ch0 < p.N;
      for (int c = 0; c < 4; ++c) {
        const int tcol = kh * 128 + c * 32;  // first token column of this chunk
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + ACC_COL + tcol, r);
        tmem_ld_wait();
        // r[j] = D[channel = lane][token j] -> transpose: buf row j = token, column = channel
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float v = __uint_as_float(r[j]) * sc;
          if (p.act == 1) v = gelu_f(v, p.gelu_tanh);
          buf[j * 32 + ((((lane >> 2) ^ (j & 7))) << 2) + (lane & 3)] = v;
        }
        __syncwarp();
        float o[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 t = *reinterpret_cast<const float4*>(buf + lane * 32 + ((q ^ (lane & 7)) << 2));
          o[4 * q] = t.x;
          o[4 * q + 1] = t.y;
          o[4 * q + 2] = t.z;
          o[4 * q + 3] = t.w;
        }
        __syncwarp();
        const int tok = tile_m * BM + tcol + lane;
        if (warp_has_channels && tok < p.M) {
          const int64_t off8 = (static_cast<int64_t>(tok) * p.N + ch0) / 8;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float ov[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) ov[k] = o[8 * q + k];
            if (p.res_fmt >= 0) {
              float rv[8];
              if (p.res_fmt == FMT_F32) load8<FMT_F32>(p.residual, off8 + q, rv);
              else if (p.res_fmt == FMT_F16) load8<FMT_F16>(p.residual, off8 + q, rv);
              else load8<FMT_BF16>(p.residual, off8 + q, rv);
#pragma unroll
              for (int k = 0; k < 8; ++k) ov[k] += rv[k];
            }
            if (p.y_fmt == FMT_F32) store8<FMT_F32>(y_out, off8 + q, ov);
            else if (p.y_fmt == FMT_F16) store8<FMT_F16>(y_out, off8 + q, ov);
            else store8<FMT_BF16>(y_out, off8 + q, ov);
          }
        }
      }
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
  const int tiles = ((M + gemm::BM - 1) / gemm::BM) * ((N + gemm::BN - 1) / gemm::BN);
  const int kb = (K + gemm::BK - 1) / gemm::BK;
  int s = 148 / (2 * tiles);  // a tile occupies a pair of SMs
  if (s > 8) s = 8;
  if (s > kb / 16) s = kb / 16;  // keep at least 16 k-blocks per split
  return s < 1 ? 1 : s;
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
    const uint32_t box[2] = {BK, BN_CTA};
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
  const int splits = a.k_splits > 1 ? a.k_splits : 1;
  const int kb_per = (kb_total + splits - 1) / splits;
  if (splits > 1 && (a.y_fmt != FMT_F32 || a.residual != nullptr || a.act != 0)) return cudaErrorInvalidValue;
  Params p{a.scale, a.y,         a.residual, a.M, a.N, a.K, a.y_fmt, a.residual ? a.res_fmt : -1,
           a.act,   a.gelu_tanh, kb_per,     static_cast<int64_t>(a.M) * a.N};
  dim3 grid(2 * ((a.M + BM - 1) / BM), (a.N + BN - 1) / BN, (kb_total + kb_per - 1) / kb_per);
  auto kern = f16 ? gemm_w8a16_kernel<true> : gemm_w8a16_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, THREADS, SMEM_BYTES, s>>>(tm_x, tm_w, p, g);
  return cudaGetLastError();
}

}  // namespace jab
