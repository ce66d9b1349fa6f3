// Y = epilogue( A (W8)^T * scale ) on the 5th-generation tensor cores.
//
// A: bf16 activations [M, K] row-major.  W8: e4m3 weights [N, K] row-major with an
// fp32 per-output-row scale, the storage of the Ideogram 4 FP8 checkpoint
// (unsloth diffusion_ideogram4.py commit log, fp8 loader commit: the real weight is
// fp8 * weight_scale[:, None]).  Both operands are K-major, so the problem is the
// "TN" GEMM tcgen05 reads natively.
//
// The checkpoint's numerics are W8 dequantised, activations 16-bit.  e4m3 is a
// subset of both bf16 and f16, so each weight tile is widened on chip, exactly,
// to the activation format (bf16, or f16 for the block's internal activations)
// and fed to tcgen05.mma kind::f16 with an fp32 accumulator in TMEM; the per-row
// scale is applied once per output in the epilogue (scale[n] * sum_k a*w8 is
// sum_k a*(w8*scale[n]) up to rounding).  The epilogue writes bf16, f16 or fp32
// and can add a bf16 / f16 / fp32 residual.
//
// CTA tile 128 x 256 x 64, one CTA per output tile.  Warp roles:
//   warp 0      TMA producer: A tile (128 x 64, 128B swizzle) and the raw W8 tile
//               (256 x 64 bytes) into a 4-stage ring.
//   warp 1      TMEM allocation; one lane issues the MMAs (4 x K=16 per stage).
//   warps 2..9  convert W8 -> 16-bit into the 128B-swizzled K-major layout the MMA
//               reads (2-stage ring; two converter warps per scheduler to hide the
//               conversion latency), then run the epilogue: tcgen05.ld of the
//               accumulator (warp w reads TMEM lanes 32*(w%4).., column half
//               (w-2)/4), scale, optional GELU / residual, stores.
#include "common.cuh"

namespace jab {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int RAW_STAGES = 4;
constexpr int CVT_STAGES = 2;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B8_BYTES = BN * BK;
constexpr int B16_BYTES = BN * BK * 2;
constexpr int THREADS = 320;
constexpr int CVT_WARPS = 8;
constexpr int TMEM_COLS = 256;

constexpr int OFF_A = 0;
constexpr int OFF_B8 = OFF_A + RAW_STAGES * A_BYTES;
constexpr int OFF_B16 = OFF_B8 + RAW_STAGES * B8_BYTES;
constexpr int OFF_SCALE = OFF_B16 + CVT_STAGES * B16_BYTES;
constexpr int OFF_BAR = OFF_SCALE + BN * 4;
constexpr int NUM_BARS = 2 * RAW_STAGES + 2 * CVT_STAGES + 2;
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
  int kb_per_split;          // k-blocks per split (grid.z splits); all of K when not split
  int64_t y_split_stride;    // elements between the fp32 partial outputs of consecutive splits
};

__device__ __forceinline__ float gelu_f(float x, int tanh_form) {
  if (tanh_form) {
    const float k0 = 0.7978845608028654f, k1 = 0.044715f;
    return 0.5f * x * (1.f + tanhf(k0 * (x + k1 * x * x * x)));
  }
  return 0.5f * x * (1.f + erff(x * 0.7071067811865476f));
}

template <bool F16>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_w8a16_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const Params p, const KernelGuard guard) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + OFF_A;
  uint8_t* sB8 = smem + OFF_B8;
  uint8_t* sB16 = smem + OFF_B16;
  float* sScale = reinterpret_cast<float*>(smem + OFF_SCALE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = bars + RAW_STAGES;
  uint64_t* cvt_full = bars + 2 * RAW_STAGES;
  uint64_t* cvt_empty = bars + 2 * RAW_STAGES + CVT_STAGES;
  uint64_t* acc_full = bars + 2 * RAW_STAGES + 2 * CVT_STAGES;
  uint64_t* drain_bar = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int tile_m = blockIdx.x;
  const int tile_n = blockIdx.y;
  const int kb_total = (p.K + BK - 1) / BK;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int num_kb = min(kb_total - kb0, p.kb_per_split);
  void* const y_out = static_cast<char*>(p.y) + blockIdx.z * p.y_split_stride * 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_STAGES; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], 1 + CVT_WARPS);  // MMA commit + converter warps
    }
    for (int c = 0; c < CVT_STAGES; ++c) {
      mbar_init(&cvt_full[c], CVT_WARPS);
      mbar_init(&cvt_empty[c], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  for (int i = threadIdx.x; i < BN; i += THREADS) {
    const int n = tile_n * BN + i;
    sScale[i] = n < p.N ? p.scale[n] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    int issued = 0;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % RAW_STAGES;
      const uint32_t it = static_cast<uint32_t>(kb / RAW_STAGES);
      if (!mbar_wait(&raw_empty[s], (it & 1u) ^ 1u, guard, abort_flag, ERR_TIMEOUT_GEMM_PRODUCER)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&raw_full[s], A_BYTES + B8_BYTES);
        tma_load_2d(sA + s * A_BYTES, &tm_a, &raw_full[s], (kb0 + kb) * BK, tile_m * BM);
        tma_load_2d(sB8 + s * B8_BYTES, &tm_b, &raw_full[s], (kb0 + kb) * BK, tile_n * BN);
      }
      __syncwarp();
      issued = kb + 1;
    }
    // Never leave with copies in flight: wait for the last load of every stage.
    for (int s = 0; s < RAW_STAGES && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / RAW_STAGES) * RAW_STAGES;
      const uint32_t it = static_cast<uint32_t>(last / RAW_STAGES);
      mbar_wait(&raw_full[s], it & 1u, guard, abort_flag, ERR_TIMEOUT_GEMM_DRAIN, true);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = idesc_f16kind(BM, BN, F16, false, false);
    bool ok = true;
    for (int kb = 0; kb < num_kb && ok; ++kb) {
      const int s = kb % RAW_STAGES;
      const int c = kb % CVT_STAGES;
      ok = mbar_wait(&raw_full[s], static_cast<uint32_t>(kb / RAW_STAGES) & 1u, guard, abort_flag,
                     ERR_TIMEOUT_GEMM_MMA) &&
           mbar_wait(&cvt_full[c], static_cast<uint32_t>(kb / CVT_STAGES) & 1u, guard, abort_flag,
                     ERR_TIMEOUT_GEMM_MMA);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a0 = smem_u32(sA + s * A_BYTES);
        const uint32_t b0 = smem_u32(sB16 + c * B16_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(a0 + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(b0 + kk * 32, 16, 1024);
          mma_f16kind_ss(tmem_acc, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        mma_commit(&raw_empty[s]);
        mma_commit(&cvt_empty[c]);
      }
      __syncwarp();
    }
    if (lane == 0) {
      if (ok) mma_commit(acc_full);
      mma_commit(drain_bar);  // all MMAs retired before TMEM is freed
    }
    __syncwarp();
    mbar_wait(drain_bar, 0u, guard, abort_flag, ERR_TIMEOUT_GEMM_DRAIN, true);
  } else {
    // ---------------- converters (warps 2..9), then the epilogue
    const int ct = threadIdx.x - 64;  // 0..255
    bool ok = true;
    for (int kb = 0; kb < num_kb && ok; ++kb) {
      const int s = kb % RAW_STAGES;
      const int c = kb % CVT_STAGES;
      ok = mbar_wait(&raw_full[s], static_cast<uint32_t>(kb / RAW_STAGES) & 1u, guard, abort_flag,
                     ERR_TIMEOUT_GEMM_CONVERT) &&
           mbar_wait(&cvt_empty[c], (static_cast<uint32_t>(kb / CVT_STAGES) & 1u) ^ 1u, guard, abort_flag,
                     ERR_TIMEOUT_GEMM_CONVERT);
      if (!ok) break;
      const uint8_t* src = sB8 + s * B8_BYTES;
      uint8_t* dst = sB16 + c * B16_BYTES;
#pragma unroll
      for (int i = 0; i < (BN * BK / 16) / (32 * CVT_WARPS); ++i) {
        const int chunk = i * (32 * CVT_WARPS) + ct;
        const int r = chunk >> 2;
        const int q = chunk & 3;
        const uint4 v = *reinterpret_cast<const uint4*>(src + r * 64 + q * 16);
        uint4 o0, o1;
        e4m3x4_to_16x4<F16>(v.x, o0.x, o0.y);
        e4m3x4_to_16x4<F16>(v.y, o0.z, o0.w);
        e4m3x4_to_16x4<F16>(v.z, o1.x, o1.y);
        e4m3x4_to_16x4<F16>(v.w, o1.z, o1.w);
        uint8_t* row = dst + r * 128;
        *reinterpret_cast<uint4*>(row + (((2 * q) ^ (r & 7)) << 4)) = o0;
        *reinterpret_cast<uint4*>(row + (((2 * q + 1) ^ (r & 7)) << 4)) = o1;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&cvt_full[c]);
        mbar_arrive(&raw_empty[s]);
      }
    }

    // ---------------- epilogue: warp (w % 4) owns TMEM lanes 32*(w%4) .. +31
    if (ok && mbar_wait(acc_full, 0u, guard, abort_flag, ERR_TIMEOUT_GEMM_EPILOGUE)) {
      tc_fence_after();
      const int quarter = warp & 3;
      const int half = (warp - 2) >> 2;
      const int row = tile_m * BM + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      for (int cc = half * (BN / 64); cc < (half + 1) * (BN / 64); ++cc) {
        const int col0 = tile_n * BN + cc * 32;
        if (col0 >= p.N) break;
        uint32_t r[32];
        tmem_ld32(tmem_acc + (static_cast<uint32_t>(quarter * 32) << 16) + cc * 32, r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) * sScale[cc * 32 + j];
        if (p.act == 1) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = gelu_f(v[j], p.gelu_tanh);
        }
        if (row_ok) {
          const int64_t off8 = (static_cast<int64_t>(row) * p.N + col0) / 8;
          if (p.res_fmt >= 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float rv[8];
              if (p.res_fmt == FMT_F32) load8<FMT_F32>(p.residual, off8 + q, rv);
              else if (p.res_fmt == FMT_F16) load8<FMT_F16>(p.residual, off8 + q, rv);
              else load8<FMT_BF16>(p.residual, off8 + q, rv);
#pragma unroll
              for (int k = 0; k < 8; ++k) v[q * 8 + k] += rv[k];
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float ov[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) ov[k] = v[q * 8 + k];
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, TMEM_COLS);
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
  int s = 148 / tiles;
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
  CUtensorMap tm_a, tm_b;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K) * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_tmap(&tm_a, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(a.a), dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K)};
    const uint32_t box[2] = {BK, BN};
    if (!make_tmap(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.w), dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  const int kb_total = (a.K + BK - 1) / BK;
  const int splits = a.k_splits > 1 ? a.k_splits : 1;
  const int kb_per = (kb_total + splits - 1) / splits;
  Params p{a.scale, a.y, a.residual, a.M, a.N, a.K, a.y_fmt, a.residual ? a.res_fmt : -1, a.act, a.gelu_tanh,
           kb_per, static_cast<int64_t>(a.M) * a.N};
  if (splits > 1 && (a.y_fmt != FMT_F32 || a.residual != nullptr || a.act != 0)) return cudaErrorInvalidValue;
  dim3 grid((a.M + BM - 1) / BM, (a.N + BN - 1) / BN, (kb_total + kb_per - 1) / kb_per);
  auto kern = f16 ? gemm_w8a16_kernel<true> : gemm_w8a16_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, THREADS, SMEM_BYTES, s>>>(tm_a, tm_b, p, g);
  return cudaGetLastError();
}

}  // namespace jab
