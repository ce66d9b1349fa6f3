// Joint bidirectional attention on the 5th-generation tensor cores.
//
// The Ideogram 4 DiT is single-stream: text and image tokens form one sequence
// through the same self-attention (Ideogram 4 deep dive, section 4-2; Ideogram 4.0
// announcement thread), so every query attends to every key with no mask:
//   O_h = softmax(q_h k_h^T / sqrt(hd)) v_h.
//
// One CTA per (batch, head, 128-query tile), flash-style over 128-key blocks:
//   warp 0      TMA producer: Q once, then K_j and V_j into a 2-stage ring, read
//               straight out of the fused qkv buffer [B, S, 3d] (3D tensor map).
//   warp 1      TMEM allocation; one lane issues S_j = Q K_j^T (kind::f16, into one
//               of two TMEM S buffers) and O += P_{j-1} V_{j-1} (P from shared
//               memory, V read MN-major), so QK^T of block j overlaps softmax j-1.
//   warps 2..5  softmax: thread i owns query row i (TMEM lane i), so the running
//               max and sum are thread-local.  exp2 with the log2(e)/sqrt(hd) scale
//               folded in; P is written as 16-bit (the q/k/v format: bf16 or f16)
//               into a 128B-swizzled K-major tile.
//               The running max is only raised (and O in TMEM rescaled) when it
//               grows by more than 2^8; until then the stale max is used for both
//               P and the row sum, which leaves O / l unchanged and keeps P <= 256.
//               The final O / l is stored in the q/k/v format.
#include "common.cuh"

namespace jab {
namespace attn {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

template <int HD>
struct Layout {
  static constexpr int SLAB = 128 * 128;  // 128 rows x 128 bytes (64 bf16)
  static constexpr int TILE = (HD / 64) * SLAB;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + 2 * TILE;
  static constexpr int OFF_P = OFF_V + 2 * TILE;
  static constexpr int OFF_BAR = OFF_P + 2 * SLAB;
  static constexpr int NUM_BARS = 16;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
};

template <int HD, int F>
__global__ void __launch_bounds__(THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm, uint16_t* __restrict__ out, int seq, int n_heads,
                     const KernelGuard guard) {
  using L = Layout<HD>;
  constexpr bool kF16 = F == FMT_F16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* kv_empty = bars + 5;  // [2]
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* s_empty = bars + 9;   // [2]
  uint64_t* p_full = bars + 11;
  uint64_t* p_empty = bars + 12;
  uint64_t* o_full = bars + 13;
  uint64_t* drain_bar = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const int q0 = blockIdx.x * BQ;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int d = n_heads * HD;
  const int nb = (seq + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(p_empty, 1);
    mbar_init(o_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm);
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem + 256;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, L::TILE);
      for (int c = 0; c < HD / 64; ++c) tma_load_3d(sQ + c * L::SLAB, &tm, q_full, head * HD + 64 * c, q0, b);
    }
    __syncwarp();
    int issued = 0;
    for (int j = 0; j < nb; ++j) {
      const int st = j & 1;
      const uint32_t it = static_cast<uint32_t>(j >> 1);
      if (!mbar_wait(&kv_empty[st], (it & 1u) ^ 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_PRODUCER)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&k_full[st], L::TILE);
        for (int c = 0; c < HD / 64; ++c)
          tma_load_3d(sK + st * L::TILE + c * L::SLAB, &tm, &k_full[st], d + head * HD + 64 * c, j * BKV, b);
        mbar_arrive_expect_tx(&v_full[st], L::TILE);
        for (int c = 0; c < HD / 64; ++c)
          tma_load_3d(sV + st * L::TILE + c * L::SLAB, &tm, &v_full[st], 2 * d + head * HD + 64 * c, j * BKV, b);
      }
      __syncwarp();
      issued = j + 1;
    }
    mbar_wait(q_full, 0u, guard, abort_flag, ERR_TIMEOUT_ATTN_DRAIN, true);
    for (int st = 0; st < 2 && st < issued; ++st) {
      const int last = st + ((issued - 1 - st) / 2) * 2;
      const uint32_t it = static_cast<uint32_t>(last >> 1);
      mbar_wait(&k_full[st], it & 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_DRAIN, true);
      mbar_wait(&v_full[st], it & 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_DRAIN, true);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc_s = idesc_f16kind(BQ, BKV, kF16, false, false);
    constexpr uint32_t idesc_o = idesc_f16kind(BQ, HD, kF16, false, true);
    bool ok = mbar_wait(q_full, 0u, guard, abort_flag, ERR_TIMEOUT_ATTN_MMA);
    auto issue_pv = [&](int i) -> bool {
      const int st = i & 1;
      if (!mbar_wait(&v_full[st], static_cast<uint32_t>(i >> 1) & 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_MMA))
        return false;
      if (!mbar_wait(p_full, static_cast<uint32_t>(i) & 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_MMA)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t pbase = smem_u32(sP);
        const uint32_t vbase = smem_u32(sV + st * L::TILE);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(pbase + (kk >> 2) * L::SLAB + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(vbase + kk * 16 * 128, L::SLAB, 1024);
          mma_f16kind_ss(tmem_o, ad, bd, idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(p_empty);
        mma_commit(&kv_empty[st]);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < nb && ok; ++j) {
      const int st = j & 1;
      ok = mbar_wait(&k_full[st], static_cast<uint32_t>(j >> 1) & 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_MMA) &&
           mbar_wait(&s_empty[st], (static_cast<uint32_t>(j >> 1) & 1u) ^ 1u, guard, abort_flag,
                     ERR_TIMEOUT_ATTN_MMA);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t qbase = smem_u32(sQ);
        const uint32_t kbase = smem_u32(sK + st * L::TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::SLAB + (kk & 3) * 32;
          mma_f16kind_ss(tmem + st * BKV, smem_desc_sw128(qbase + off, 16, 1024), smem_desc_sw128(kbase + off, 16, 1024),
                      idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[st]);
      }
      __syncwarp();
      if (j > 0) ok = issue_pv(j - 1);
    }
    if (ok) ok = issue_pv(nb - 1);
    if (lane == 0) {
      if (ok) mma_commit(o_full);
      mma_commit(drain_bar);
    }
    __syncwarp();
    mbar_wait(drain_bar, 0u, guard, abort_flag, ERR_TIMEOUT_ATTN_DRAIN, true);
  } else {
    // ---------------- softmax (warps 2..5): thread owns query row 32*(warp%4) + lane
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
    float m_used = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nb && ok; ++j) {
      const int st = j & 1;
      if (!mbar_wait(&s_full[st], static_cast<uint32_t>(j >> 1) & 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_SOFTMAX)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_off + st * BKV + 32 * c, raw);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k) s[32 * c + k] = __uint_as_float(raw[k]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[st]);

      const int valid = seq - j * BKV;  // keys beyond the sequence are masked
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < BKV; ++k) {
        s[k] = k < valid ? s[k] * c_log2 : -INFINITY;
        mx = fmaxf(mx, s[k]);
      }
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_used + RESCALE_THRESHOLD) {
        alpha = ex2_approx(m_used - mx);  // 0 on the first block
        m_used = mx;
        rescale = true;
      }
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < BKV; ++k) {
        s[k] = ex2_approx(s[k] - m_used);
        sum += s[k];
      }
      l = l * alpha + sum;

      // PV of the previous block must be done: P buffer free, O current.
      if (j > 0 &&
          !mbar_wait(p_empty, static_cast<uint32_t>(j - 1) & 1u, guard, abort_flag, ERR_TIMEOUT_ATTN_SOFTMAX)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(tmem_o + lane_off + 32 * c, raw);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) raw[k] = __float_as_uint(__uint_as_float(raw[k]) * alpha);
          tmem_st32(tmem_o + lane_off + 32 * c, raw);
        }
        tmem_st_wait();
      }
      // P row -> 16-bit, 128B-swizzled K-major (two 64-key slabs)
#pragma unroll
      for (int kc = 0; kc < BKV / 8; ++kc) {
        uint4 o;
        o.x = pack2<F>(s[8 * kc + 0], s[8 * kc + 1]);
        o.y = pack2<F>(s[8 * kc + 2], s[8 * kc + 3]);
        o.z = pack2<F>(s[8 * kc + 4], s[8 * kc + 5]);
        o.w = pack2<F>(s[8 * kc + 6], s[8 * kc + 7]);
        uint8_t* dst = sP + (kc >> 3) * L::SLAB + r * 128 + ((((kc & 7) ^ (r & 7))) << 4);
        *reinterpret_cast<uint4*>(dst) = o;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(o_full, 0u, guard, abort_flag, ERR_TIMEOUT_ATTN_SOFTMAX)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int row = q0 + r;
      uint16_t* dst = out + (static_cast<size_t>(b) * seq + row) * d + head * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(tmem_o + lane_off + 32 * c, raw);
        tmem_ld_wait();
        if (row < seq) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = pack2<F>(__uint_as_float(raw[8 * q + 0]) * inv_l, __uint_as_float(raw[8 * q + 1]) * inv_l);
            o.y = pack2<F>(__uint_as_float(raw[8 * q + 2]) * inv_l, __uint_as_float(raw[8 * q + 3]) * inv_l);
            o.z = pack2<F>(__uint_as_float(raw[8 * q + 4]) * inv_l, __uint_as_float(raw[8 * q + 5]) * inv_l);
            o.w = pack2<F>(__uint_as_float(raw[8 * q + 6]) * inv_l, __uint_as_float(raw[8 * q + 7]) * inv_l);
            reinterpret_cast<uint4*>(dst + 32 * c)[q] = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int HD, int F>
cudaError_t launch_hd(const CUtensorMap& tm, void* out, int batch, int seq, int n_heads, const KernelGuard& g,
                      cudaStream_t s) {
  using L = Layout<HD>;
  cudaError_t e =
      cudaFuncSetAttribute(attention_kernel<HD, F>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((seq + BQ - 1) / BQ, n_heads, batch);
  attention_kernel<HD, F><<<grid, THREADS, L::SMEM, s>>>(tm, static_cast<uint16_t*>(out), seq, n_heads, g);
  return cudaGetLastError();
}

}  // namespace attn

cudaError_t launch_attention(const void* qkv, void* out, int fmt, int batch, int seq, int n_heads, int head_dim,
                             const KernelGuard& g, cudaStream_t s) {
  if (batch <= 0 || seq <= 0) return cudaSuccess;
  if (fmt != FMT_BF16 && fmt != FMT_F16) return cudaErrorInvalidValue;
  const int d = n_heads * head_dim;
  CUtensorMap tm;
  const uint64_t dims[3] = {static_cast<uint64_t>(3 * d), static_cast<uint64_t>(seq), static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(3 * d) * 2, static_cast<uint64_t>(seq) * 3 * d * 2};
  const uint32_t box[3] = {64, attn::BKV, 1};
  if (!make_tmap(&tm, fmt == FMT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                 const_cast<void*>(qkv), dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (head_dim == 128)
    return fmt == FMT_F16 ? attn::launch_hd<128, FMT_F16>(tm, out, batch, seq, n_heads, g, s)
                          : attn::launch_hd<128, FMT_BF16>(tm, out, batch, seq, n_heads, g, s);
  if (head_dim == 64)
    return fmt == FMT_F16 ? attn::launch_hd<64, FMT_F16>(tm, out, batch, seq, n_heads, g, s)
                          : attn::launch_hd<64, FMT_BF16>(tm, out, batch, seq, n_heads, g, s);
  return cudaErrorInvalidValue;
}

}  // namespace jab
