// Y = act( (A8 W8^T) * sa[m] * sw[n] ) with FP8 activations and FP8 weights, on the
// 5th-generation tensor cores (tcgen05.mma kind::f8f6f4, e4m3 x e4m3, fp32 accumulator).
//
// The W8A8 variant of the block GEMMs whose inputs come straight from a norm (the QKV and
// MLP-up projections): A8 holds per-token e4m3 codes with an fp32 scale per row, W8 the
// checkpoint's e4m3 weights with their per-output-row weight_scale (unsloth
// diffusion_ideogram4.py commit log, fp8 loader commit).  Both scales are applied once per
// output in the epilogue.  With both operands 8-bit the tensor core runs at twice the 16-bit
// rate and no widening is needed: TMA writes the operand tiles the MMA reads.
//
// Two CTAs on two SMs (a cluster of 2) share a 256-token x 512-channel tile through the pair
// MMA (M = 256, N = 256, issued into two TMEM accumulators = all 512 columns), like the W8A16
// kernel.  Per CTA and K-step of 128: its 128 tokens of A (16 KB) and its 2 x 128 weight rows
// (32 KB), 128-byte swizzle, all counted on the leader's barrier; 3-stage ring.  Persistent: one
// CTA pair per SM pair walks the work units.
//   warp 0      TMA producer (runs ahead across units, bounded by the ring)
//   warp 1      TMEM allocation; in the leader one lane issues 2 x 4 pair MMAs per stage
//   warps 2..9  epilogue: warp w reads TMEM lanes 32 (w % 4).., accumulator (w - 2) / 4; per
//               32-channel chunk it scales (and applies GELU), packs a swizzled 32 x 32 box and
//               hands it to a TMA store.  After the unit's last TMEM read the warps release the
//               accumulators (a barrier in the leader) so the next unit's MMAs start while the
//               last stores drain.  No TMA load is multicast.
#include <string.h>

#include "common.cuh"

namespace jab {
namespace gemm8 {

constexpr int BM = 256;
constexpr int BM_CTA = 128;
constexpr int BN = 512;
constexpr int BN_MMA = 256;
constexpr int BK = 128;  // K elements (= bytes) per stage
constexpr int STAGES = 3;
constexpr int A_BYTES = BM_CTA * BK;
constexpr int W_BLOCK = 128 * BK;
constexpr int W_BYTES = 2 * W_BLOCK;
constexpr int STAGE_BYTES = A_BYTES + W_BYTES;
constexpr int THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr int TMEM_COLS = 512;
constexpr int MAX_PAIRS = 74;
constexpr int EPI_WARP_BYTES = 8 * 1024;  // two 32 x 32 output boxes (4 KB each at fp32)
constexpr int OFF_EPI = STAGES * STAGE_BYTES;
constexpr int OFF_SCALE = OFF_EPI + EPI_WARPS * EPI_WARP_BYTES;
constexpr int OFF_BAR = OFF_SCALE + EPI_WARPS * BN_MMA * 4;
constexpr int NUM_BARS = 2 * STAGES + 3;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

struct Params {
  const float* sa;  // [M] per-token activation scales
  const float* sw;  // [N] per-row weight scales
  int M, N, K;
  int y_fmt;  // FMT_BF16 / FMT_F16 / FMT_F32
  int act;    // 0 none, 1 GELU
  int gelu_tanh;
  int tiles_m, tiles_n, units;
  int y_evict_first;
};

// GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) = x / (1 + exp(-2y)).  The exact
// form is gelu_erf_pair (common.cuh).
__device__ __forceinline__ float gelu_tanh(float x) {
  const float y = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
  return x * rcp_approx(1.f + ex2_approx(-2.8853900817779268f * y));
}

// D[tmem] (+)= A * B^T, kind::f8f6f4 (e4m3 x e4m3), issued by the leader for the pair.
__device__ __forceinline__ void mma_f8_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_y, const Params p, const KernelGuard guard) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;                  // [STAGES] leader: both CTAs' A and W tiles landed
  uint64_t* empty = full + STAGES;        // [STAGES] the stage's MMAs are done
  uint64_t* acc_full = empty + STAGES;    // one phase per unit
  uint64_t* acc_empty = acc_full + 1;     // leader: both CTAs' epilogue warps have read TMEM
  uint64_t* drain_bar = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;
  const int kb_total = (p.K + BK - 1) / BK;
  auto unit_mn = [&](int u, int& tile_m, int& tile_n) {
    tile_m = u % p.tiles_m;
    tile_n = u / p.tiles_m;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * EPI_WARPS);
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_y);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_then_release();

  if (warp == 0) {
    // ---------------- TMA producer
    int g = 0;
    bool ok = true;
    for (int u = pair; u < p.units && ok; u += pairs) {
      int tile_m, tile_n;
      unit_mn(u, tile_m, tile_n);
      const int tok = tile_m * BM + static_cast<int>(rank) * BM_CTA;
      const int wr = tile_n * BN + static_cast<int>(rank) * 128;  // block b adds b * 256
      for (int kb = 0; kb < kb_total; ++kb) {
        const int s = g % STAGES;
        if (!mbar_wait(&empty[s], (static_cast<uint32_t>(g / STAGES) & 1u) ^ 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_GEMM_PRODUCER, rank, g))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* st = smem + s * STAGE_BYTES;
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          tma_load_2d_pair(st, &tm_a, bar, kb * BK, tok);
          tma_load_2d_pair(st + A_BYTES, &tm_w, bar, kb * BK, wr);
          tma_load_2d_pair(st + A_BYTES + W_BLOCK, &tm_w, bar, kb * BK, wr + BN_MMA);
        }
        __syncwarp();
        ++g;
      }
    }
    if (leader) {  // the leader's barriers count both CTAs' copies; the peer waits at the cluster barrier
      for (int s = 0; s < STAGES && s < g; ++s) {
        const int last = s + ((g - 1 - s) / STAGES) * STAGES;
        mbar_wait(&full[s], static_cast<uint32_t>(last / STAGES) & 1u, guard, abort_flag,
                  where_code(ERR_TIMEOUT_GEMM_DRAIN, rank, s), true);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only)
    if (leader) {
      constexpr uint32_t idesc = idesc_f16kind(BM, BN_MMA, true, false, false);  // type code 0 = e4m3 here
      bool ok = true;
      int g = 0, ui = 0;
      for (int u = pair; u < p.units && ok; u += pairs, ++ui) {
        if (ui > 0 && !mbar_wait(acc_empty, static_cast<uint32_t>(ui - 1) & 1u, guard, abort_flag,
                                 where_code(ERR_TIMEOUT_GEMM_MMA_X, rank, ui))) {
          ok = false;
          break;
        }
        for (int kb = 0; kb < kb_total; ++kb) {
          const int s = g % STAGES;
          if (!mbar_wait(&full[s], static_cast<uint32_t>(g / STAGES) & 1u, guard, abort_flag,
                         where_code(ERR_TIMEOUT_GEMM_MMA, rank, g))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t w0 = a0 + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk) {
              const uint64_t ad = smem_desc_sw128(a0 + kk * 32, 16, 1024);
#pragma unroll
              for (int b = 0; b < 2; ++b)
                mma_f8_ss_pair(tmem + b * BN_MMA, ad, smem_desc_sw128(w0 + b * W_BLOCK + kk * 32, 16, 1024), idesc,
                               (kb | kk) != 0 ? 1u : 0u);
            }
            mma_commit_pair(&empty[s], 0x3);
            if (kb + 1 == kb_total) mma_commit_pair(acc_full, 0x3);
          }
          __syncwarp();
          ++g;
        }
      }
      if (lane == 0) mma_commit_pair(drain_bar, 0x3);
      __syncwarp();
    }
    mbar_wait(drain_bar, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_GEMM_DRAIN_MMA, rank, 0), true);
  } else {
    // ---------------- epilogue (warps 2..9)
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int acc = ew >> 2;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN_MMA;
    float* sScale = reinterpret_cast<float*>(smem + OFF_SCALE) + ew * BN_MMA;
    const int out_box = 32 * 32 * (p.y_fmt == FMT_F32 ? 4 : 2);
    uint8_t* ebox = smem + OFF_EPI + ew * EPI_WARP_BYTES;
    const uint32_t empty_bar = mapa_shared(smem_u32(acc_empty), 0);
    const uint64_t policy = l2_evict_first_policy();
    bool ok = true;
    int ui = 0;
    for (int u = pair; u < p.units && ok; u += pairs, ++ui) {
      int tile_m, tile_n;
      unit_mn(u, tile_m, tile_n);
      const int tok_warp = tile_m * BM + static_cast<int>(rank) * BM_CTA + quarter * 32;
      const int ch_warp = tile_n * BN + acc * BN_MMA;
      const int nch = tok_warp < p.M ? min(BN_MMA, p.N - ch_warp) / 32 : 0;
      {
        const int n0 = ch_warp + 8 * lane;
#pragma unroll
        for (int k = 0; k < 8; ++k) sScale[8 * lane + k] = n0 + k < p.N ? p.sw[n0 + k] : 0.f;
      }
      const int row = tok_warp + lane;
      const float sa = row < p.M ? p.sa[row] : 0.f;
      if (!mbar_wait(acc_full, static_cast<uint32_t>(ui) & 1u, guard, abort_flag,
                     where_code(ERR_TIMEOUT_GEMM_EPILOGUE, rank, ui))) {
        ok = false;
        break;
      }
      tc_fence_after();
      __syncwarp();
      for (int c = 0; c < BN_MMA / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(taddr + 32 * c, rr);
        tmem_ld_wait();
        if (c == BN_MMA / 32 - 1) {  // this warp's last TMEM read of the unit: release the accumulators
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(empty_bar);
        }
        if (c >= nch) continue;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(rr[j]) * (sScale[32 * c + j] * sa);
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
        if (lane == 0) bulk_wait_group_read<1>();  // the box written two chunks ago has been read
        __syncwarp();
        uint8_t* orow = ebox + (c & 1) * out_box;
        if (p.y_fmt == FMT_F32) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(orow + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
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
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (p.y_evict_first)
            tma_store_3d_hint(&tm_y, orow, ch_warp + 32 * c, tok_warp, 0, policy);
          else
            tma_store_3d(&tm_y, orow, ch_warp + 32 * c, tok_warp, 0);
          bulk_commit_group();
        }
      }
      if (lane == 0) bulk_wait_group_read<0>();  // the boxes are free before the next unit writes them
      __syncwarp();
    }
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace gemm8

cudaError_t launch_gemm_w8a8(const GemmArgs8& a, const KernelGuard& g, cudaStream_t s) {
  using namespace gemm8;
  if (a.M <= 0 || a.N <= 0) return cudaSuccess;
  if (a.N % 32 != 0 || a.K % 16 != 0) return cudaErrorInvalidValue;
  CUtensorMap tm_a, tm_w, tm_y;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K)};
    const uint32_t box[2] = {BK, 128};
    if (!make_tmap(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.w), dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(a.K), static_cast<uint64_t>(a.M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.K)};
    const uint32_t box[2] = {BK, BM_CTA};
    if (!make_tmap(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.a), dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t esz = a.y_fmt == FMT_F32 ? 4 : 2;
    const uint64_t dims[3] = {static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M), 1};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.N) * esz, static_cast<uint64_t>(a.N) * a.M * esz};
    const uint32_t box[3] = {32, 32, 1};
    const CUtensorMapDataType dt = a.y_fmt == FMT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : (a.y_fmt == FMT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    if (!make_tmap(&tm_y, dt, 3, a.y, dims, strides, box,
                   a.y_fmt == FMT_F32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  const int tiles_m = (a.M + BM - 1) / BM, tiles_n = (a.N + BN - 1) / BN;
  const int units = tiles_m * tiles_n;
  const int64_t y_bytes = static_cast<int64_t>(a.M) * a.N * (a.y_fmt == FMT_F32 ? 4 : 2);
  Params p{a.sa, a.sw, a.M, a.N, a.K, a.y_fmt, a.act, a.gelu_tanh, tiles_m, tiles_n, units,
           y_bytes > (100ll << 20) ? 1 : 0};
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 2 * MAX_PAIRS;
  const int pairs = min(units, max(1, sms / 2));
  cudaError_t e = cudaFuncSetAttribute(gemm_w8a8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  e = launch_pdl(gemm_w8a8_kernel, dim3(2 * pairs), dim3(THREADS), SMEM_BYTES, s, tm_a, tm_w, tm_y, p, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace jab
