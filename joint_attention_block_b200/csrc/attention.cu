// Joint bidirectional attention on the 5th-generation tensor cores.
//
// The Ideogram 4 DiT is single-stream: text and image tokens form one sequence
// through the same self-attention (Ideogram 4 deep dive, section 4-2; Ideogram 4.0
// announcement thread), so every query attends to every key with no mask:
//   O_h = softmax(q_h k_h^T / sqrt(hd)) v_h.
// A batch of prompts padded to one length passes a per-element key count; keys at or
// beyond it are left out of every row's softmax (padding sits at the end of each element).
//
// Two CTAs on two SMs (a cluster of 2) share 256 queries of one (batch, head): each CTA
// holds 128 query rows, and the pair form of the MMA (tcgen05.mma.cta_group::2, M = 256)
// lets each CTA load only half of every key/value block:
//   S = Q K^T    N = 128 keys; CTA r loads keys [64 r, 64 r + 64) of the block
//   O += P V     N = hd;      CTA r loads value columns [r hd/2, (r + 1) hd/2) of all 128 keys,
//                             P (the A operand) is read from each CTA's own tensor memory.
// The key blocks are processed by two independent groups: group 0 takes the even blocks,
// group 1 the odd ones, each with its own S buffer, O accumulator and running max/sum in
// TMEM (S0 | S1 | O0 | O1 = 512 columns for hd 128).  While one group's softmax runs, the
// tensor core computes the other group's P V and next S, so the exponentials of one group
// overlap the MMAs of the other.  At the end the two partial results of each row are merged
// (a two-way split of the keys, combined with their maxima and sums).
//
//   warp 0       TMA producer: this CTA's Q rows once, then per key block its K and V halves
//                (4-stage ring), straight from the fused qkv buffer [B, S, 3d]; every copy
//                completes on the leader CTA's barriers.
//   warp 1       TMEM allocation (pair); in the leader, one lane issues
//                S(0), S(1), then per block j: P V(j) into O_{j%2}, S(j+2) into S_{j%2}.
//   warps 2..5   softmax of group 0, warps 6..9 of group 1; thread = query row (TMEM lane),
//                so the running max and sum are thread-local.  The whole row of S comes out of
//                TMEM in one round trip; exp2 with log2(e)/sqrt(hd) folded in (packed fp32 pair
//                arithmetic for the scaling and the sums); P is written back over S as 16-bit
//                pairs.  The max in use is only raised (and O rescaled in TMEM) when a block
//                exceeds it by 2^8, which leaves O / l unchanged and keeps P <= 256.
//                At the end both groups merge the two partial results, each writing half of
//                the head's columns.
#include "common.cuh"

namespace jab {
namespace attn {

constexpr int BQ = 128;   // query rows per CTA (256 per pair)
constexpr int BKV = 128;  // keys per block
constexpr int STAGES = 4;
constexpr int THREADS = 320;
constexpr int TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
#ifndef JAB_ATTN_POLY_EVERY
#define JAB_ATTN_POLY_EVERY 0
#endif
// 0: every exp2 on the MUFU unit; n > 0: one key pair in n on the FMA pipe (exp2_poly).
constexpr int POLY_EVERY = JAB_ATTN_POLY_EVERY;

template <int HD>
struct Layout {
  static constexpr int Q_SLAB = 128 * 128;  // 128 rows x 64 16-bit values, 128-byte swizzle
  static constexpr int Q_BYTES = (HD / 64) * Q_SLAB;
  static constexpr int K_SLAB = 64 * 128;  // 64 keys x 64 16-bit values
  static constexpr int K_BYTES = (HD / 64) * K_SLAB;
  static constexpr int V_ROW = HD;  // bytes per key of this CTA's hd/2 value columns
  static constexpr int V_BYTES = BKV * V_ROW;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * V_BYTES;
  static constexpr int NUM_BARS = 1 + 3 * STAGES + 6;
  static constexpr int OFF_XCH = OFF_BAR + NUM_BARS * 8;  // [group][m, l][row] fp32
  static constexpr int OFF_MISC = OFF_XCH + 2 * 2 * BQ * 4;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static_assert(OFF_V % 1024 == 0 && V_BYTES % 1024 == 0, "swizzled tiles keep 1024-byte alignment");
};

// 2^x on the FMA pipe, for x <= 8: x = n + f with n = round(x), f in [-1/2, 1/2];
// 2^f by a degree-3 polynomial (coefficients fitted to 2^f on [-1/2, 1/2] by
// iteratively reweighted least squares on Chebyshev nodes; max relative error
// 7.5e-5, below the f16 rounding of P); 2^n by adding n to the exponent field.
// Adding 1.5 * 2^23 rounds x to an integer held in the low mantissa bits, and
// (bits(t) << 23) adds exactly n << 23 because the constant's low 9 bits are 0.
// x is clamped at -125: 2^f can sit just below 1 (exponent field 126), so n must
// stay >= -125 for the exponent field to stay positive; 2^-125 is 0 in f16/bf16 P
// and masked keys (x = -inf) come out as that.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float magic = 12582912.0f;  // 1.5 * 2^23
  const float t = x + magic;
  const float n = t - magic;
  const float f = x - n;
  float p = 0.05517163500189781f;
  p = fmaf(p, f, 0.2426111251115799f);
  p = fmaf(p, f, 0.6932609677314758f);
  p = fmaf(p, f, 0.9999280571937561f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// max(a, b, c) in one instruction (three-input form of max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Barrier among the 256 softmax threads (warps 2..9) only.
__device__ __forceinline__ void softmax_bar_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <int HD, int F>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out, int seq, int n_heads,
                     const int32_t* __restrict__ kv_len, const KernelGuard guard) {
  using L = Layout<HD>;
  constexpr bool kF16 = F == FMT_F16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;                  // leader: both CTAs' Q rows landed
  uint64_t* k_full = q_full + 1;            // [STAGES] leader: both K halves of a block landed
  uint64_t* v_full = k_full + STAGES;       // [STAGES] leader: both V halves landed
  uint64_t* kv_empty = v_full + STAGES;     // [STAGES] the block's last MMA (P V) is done
  uint64_t* s_full = kv_empty + STAGES;     // [2 groups] S ready (all earlier MMAs done)
  uint64_t* p_full = s_full + 2;            // [2 groups] leader: both CTAs' P written
  uint64_t* o_full = p_full + 2;            // every MMA done
  uint64_t* drain_bar = o_full + 1;
  float* xch = reinterpret_cast<float*>(smem + L::OFF_XCH);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int q0 = (blockIdx.x >> 1) * 2 * BQ + static_cast<int>(rank) * BQ;  // this CTA's first query row
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int d = n_heads * HD;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], 8);  // 4 softmax warps of the group in each CTA
    }
    mbar_init(o_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_then_release();  // the setup above overlaps the previous kernel's tail

  // keys of this batch element: all of them, or its key count (clamped to [1, seq])
  const int nkv = kv_len == nullptr ? seq : min(max(kv_len[b], 1), seq);
  const int nb = (nkv + BKV - 1) / BKV;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      if (leader) mbar_arrive_expect_tx(q_full, 2 * L::Q_BYTES);
      const uint32_t qbar = mapa_shared(smem_u32(q_full), 0);
      for (int c = 0; c < HD / 64; ++c) tma_load_3d_pair(sQ + c * L::Q_SLAB, &tm_q, qbar, head * HD + 64 * c, q0, b);
    }
    __syncwarp();
    int issued = 0;
    for (int j = 0; j < nb; ++j) {
      const int st = j % STAGES;
      const uint32_t it = static_cast<uint32_t>(j / STAGES);
      if (!mbar_wait(&kv_empty[st], (it & 1u) ^ 1u, guard, abort_flag,
                     where_code(ERR_TIMEOUT_ATTN_PRODUCER, rank, j)))
        break;
      if (lane == 0) {
        if (leader) {
          mbar_arrive_expect_tx(&k_full[st], 2 * L::K_BYTES);
          mbar_arrive_expect_tx(&v_full[st], 2 * L::V_BYTES);
        }
        const uint32_t kbar = mapa_shared(smem_u32(&k_full[st]), 0);
        const uint32_t vbar = mapa_shared(smem_u32(&v_full[st]), 0);
        for (int c = 0; c < HD / 64; ++c)
          tma_load_3d_pair(sK + st * L::K_BYTES + c * L::K_SLAB, &tm_k, kbar, d + head * HD + 64 * c,
                           j * BKV + 64 * static_cast<int>(rank), b);
        tma_load_3d_pair(sV + st * L::V_BYTES, &tm_v, vbar, 2 * d + head * HD + static_cast<int>(rank) * (HD / 2),
                         j * BKV, b);
      }
      __syncwarp();
      issued = j + 1;
    }
    // Never leave with copies in flight: the leader's barriers count both CTAs' copies, and
    // the peer is held by the final cluster barrier until the leader has drained.
    if (leader) {
      mbar_wait(q_full, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_DRAIN, rank, 0), true);
      for (int st = 0; st < STAGES && st < issued; ++st) {
        const int last = st + ((issued - 1 - st) / STAGES) * STAGES;
        const uint32_t par = static_cast<uint32_t>(last / STAGES) & 1u;
        mbar_wait(&k_full[st], par, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_DRAIN, rank, last), true);
        mbar_wait(&v_full[st], par, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_DRAIN, rank, last), true);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only)
    if (leader) {
      constexpr uint32_t idesc_s = idesc_f16kind(2 * BQ, BKV, kF16, false, false);
      constexpr uint32_t idesc_o = idesc_f16kind(2 * BQ, HD, kF16, false, true);
      auto issue_s = [&](int j) {  // S(j) = Q K_j^T into S_{j%2}
        const int g = j & 1;
        const uint32_t qbase = smem_u32(sQ);
        const uint32_t kbase = smem_u32(sK + (j % STAGES) * L::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t oq = (kk >> 2) * L::Q_SLAB + (kk & 3) * 32;
          const uint32_t ok_ = (kk >> 2) * L::K_SLAB + (kk & 3) * 32;
          mma_f16kind_ss_pair(tmem + 128 * g, smem_desc_sw128(qbase + oq, 16, 1024),
                              smem_desc_sw128(kbase + ok_, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit_pair(&s_full[g], 0x3);
      };
      auto issue_pv = [&](int j) {  // O_{j%2} += P(j) V_j, P from TMEM (the first 64 columns of S_{j%2})
        const int g = j & 1;
        const uint32_t vbase = smem_u32(sV + (j % STAGES) * L::V_BYTES);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint32_t a = vbase + kk * 16 * L::V_ROW;
          const uint64_t bd = HD == 128 ? smem_desc_sw128(a, 16, 8 * L::V_ROW) : smem_desc_sw64(a, 16, 8 * L::V_ROW);
          mma_f16kind_ts_pair(tmem + 256 + HD * g, tmem + 128 * g + 8 * kk, bd, idesc_o,
                              (j >= 2 || kk > 0) ? 1u : 0u);
        }
        mma_commit_pair(&kv_empty[j % STAGES], 0x3);  // K_j and V_j fully consumed
      };
      bool ok = mbar_wait(q_full, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_MMA, rank, 0));
      for (int j = 0; j < 2 && j < nb && ok; ++j) {
        ok = mbar_wait(&k_full[j], 0u, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_MMA, rank, j));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) issue_s(j);
        __syncwarp();
      }
      for (int j = 0; j < nb && ok; ++j) {
        const int g = j & 1;
        ok = mbar_wait(&v_full[j % STAGES], static_cast<uint32_t>(j / STAGES) & 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_ATTN_MMA, rank, j)) &&
             mbar_wait(&p_full[g], static_cast<uint32_t>(j >> 1) & 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_ATTN_MMA, 2 + g, j));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) issue_pv(j);
        __syncwarp();
        if (j + 2 < nb) {
          // S(j+2) overwrites P(j) only after P V(j) has read it (MMAs run in issue order)
          ok = mbar_wait(&k_full[(j + 2) % STAGES], static_cast<uint32_t>((j + 2) / STAGES) & 1u, guard, abort_flag,
                         where_code(ERR_TIMEOUT_ATTN_MMA, 4 + g, j));
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) issue_s(j + 2);
          __syncwarp();
        }
      }
      if (lane == 0) {
        if (ok) mma_commit_pair(o_full, 0x3);
        mma_commit_pair(drain_bar, 0x3);  // all MMAs retired before either CTA frees TMEM
      }
      __syncwarp();
    }
    mbar_wait(drain_bar, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_DRAIN, rank, 1), true);
  } else {
    // ---------------- softmax: warps 2..5 -> group 0 (even key blocks), 6..9 -> group 1 (odd)
    const int g = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_col = tmem + lane_off + 128 * g;
    const uint32_t o_col = tmem + lane_off + 256 + HD * g;
    const uint32_t pbar = mapa_shared(smem_u32(&p_full[g]), 0);
    const float c_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
    float m_used = -INFINITY;
    float l = 0.f;
    bool ok = true;
    int i = 0;
    for (int j = g; j < nb; j += 2, ++i) {
      if (!mbar_wait(&s_full[g], static_cast<uint32_t>(i) & 1u, guard, abort_flag,
                     where_code(ERR_TIMEOUT_ATTN_SOFTMAX, rank * 2 + g, j))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int valid = nkv - j * BKV;  // keys beyond this element's key count are masked
      const bool full = valid >= BKV;    // every block but possibly the last
      // The whole row of S (128 keys) comes out of TMEM in one round trip; the max and the
      // exponentials then run from registers with independent partial results.
      uint32_t s0[32], s1[32], s2[32], s3[32];
      tmem_ld32(s_col, s0);
      tmem_ld32(s_col + 32, s1);
      tmem_ld32(s_col + 64, s2);
      tmem_ld32(s_col + 96, s3);
      tmem_ld_wait_regs(s0);
      tmem_ld_wait_regs(s1);
      tmem_ld_wait_regs(s2);
      tmem_ld_wait_regs(s3);
      float v[BKV];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        v[k] = __uint_as_float(s0[k]);
        v[32 + k] = __uint_as_float(s1[k]);
        v[64 + k] = __uint_as_float(s2[k]);
        v[96 + k] = __uint_as_float(s3[k]);
      }
      if (!full) {
#pragma unroll
        for (int k = 0; k < BKV; ++k) v[k] = k < valid ? v[k] : -INFINITY;
      }
      // row max: 8 independent chains of three-input maxima, then a short tree
      float m8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = fmax3(v[k], v[8 + k], v[16 + k]);
#pragma unroll
      for (int q = 24; q < BKV - 8; q += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = fmax3(m8[k], v[q + k], v[q + 8 + k]);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], v[BKV - 8 + k]);
      const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * c_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_used + RESCALE_THRESHOLD) {
        alpha = ex2_approx(m_used - mx);  // 0 on the group's first block
        m_used = mx;
        rescale = true;
      }
      // exponentiate, sum, and write P as 16-bit pairs over the first 64 columns of S
      float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 c2 = make_float2(c_log2, c_log2);
      const float2 nm2 = make_float2(-m_used, -m_used);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int k2 = 0; k2 < 64; k2 += 2) {
          const int k = 64 * h + k2;
          const float2 x = fma2(make_float2(v[k], v[k + 1]), c2, nm2);  // packed pair: s c - m
          float2 e;
          bool poly = false;
          if constexpr (POLY_EVERY > 0) poly = (k >> 1) % (POLY_EVERY > 0 ? POLY_EVERY : 1) == POLY_EVERY - 1;
          if (poly) {
            e.x = exp2_poly(x.x);
            e.y = exp2_poly(x.y);
          } else {
            e.x = ex2_approx(x.x);
            e.y = ex2_approx(x.y);
          }
          ps[(k2 >> 1) & 3] = add2(ps[(k2 >> 1) & 3], e);
          pk[k2 >> 1] = pack2<F>(e.x, e.y);
        }
        tmem_st32(s_col + 32 * h, pk);
      }
      const float2 ps01 = add2(ps[0], ps[1]), ps23 = add2(ps[2], ps[3]);
      const float2 ps03 = add2(ps01, ps23);
      const float sum = ps03.x + ps03.y;
      // O of this group is up to date here: its last P V was issued before S(j), and the
      // commit behind s_full covers every earlier MMA.
      if (i > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(o_col + 32 * c, raw);
          tmem_ld_wait_regs(raw);
#pragma unroll
          for (int k = 0; k < 32; ++k) raw[k] = __float_as_uint(__uint_as_float(raw[k]) * alpha);
          tmem_st32(o_col + 32 * c, raw);
        }
      }
      l = l * alpha + sum;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(pbar);
    }
    // ---- merge the two groups' partial results: each group writes half of the head's columns
    if (ok) ok = mbar_wait(o_full, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_SOFTMAX, 4 + rank, 0));
    xch[(2 * g) * BQ + r] = m_used;
    xch[(2 * g + 1) * BQ + r] = l;
    softmax_bar_sync();  // every softmax thread gets here exactly once, failed waits included
    const float mA = xch[r], lA = xch[BQ + r], mB = xch[2 * BQ + r], lB = xch[3 * BQ + r];
    const bool hasB = nb >= 2;  // group 1 saw at least one block
    if (ok) {
      tc_fence_after();
      const float m = hasB ? fmaxf(mA, mB) : mA;
      const float aA = ex2_approx(mA - m);
      const float aB = hasB ? ex2_approx(mB - m) : 0.f;
      const float inv = 1.f / (lA * aA + lB * aB);
      const float fA = aA * inv, fB = aB * inv;
      const int row = q0 + r;
      uint16_t* dst = out + (static_cast<size_t>(b) * seq + row) * d + head * HD;
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
        const int col = g * (HD / 2) + 32 * c;
        uint32_t ra[32], rb[32];
        tmem_ld32(tmem + lane_off + 256 + col, ra);
        if (hasB) tmem_ld32(tmem + lane_off + 256 + HD + col, rb);
        tmem_ld_wait_regs(ra);
        if (hasB) {
          tmem_ld_wait_regs(rb);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) rb[k] = 0u;
        }
        if (row < seq) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float o[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              o[k] = fmaf(__uint_as_float(ra[8 * q + k]), fA, __uint_as_float(rb[8 * q + k]) * fB);
            store8<F>(dst + col, q, o);
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

template <int HD, int F>
cudaError_t launch_hd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* out, int batch,
                      int seq, int n_heads, const int32_t* kv_len, const KernelGuard& g, cudaStream_t s) {
  using L = Layout<HD>;
  cudaError_t e =
      cudaFuncSetAttribute(attention_kernel<HD, F>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(2 * ((seq + 2 * BQ - 1) / (2 * BQ)), n_heads, batch);
  e = launch_pdl(attention_kernel<HD, F>, grid, dim3(THREADS), L::SMEM, s, tq, tk, tv, static_cast<uint16_t*>(out),
                 seq, n_heads, kv_len, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace attn

cudaError_t launch_attention(const void* qkv, void* out, int fmt, int batch, int seq, int n_heads, int head_dim,
                             const int32_t* kv_len, const KernelGuard& g, cudaStream_t s) {
  if (batch <= 0 || seq <= 0) return cudaSuccess;
  if (fmt != FMT_BF16 && fmt != FMT_F16) return cudaErrorInvalidValue;
  if (head_dim != 64 && head_dim != 128) return cudaErrorInvalidValue;
  const int d = n_heads * head_dim;
  const CUtensorMapDataType dt = fmt == FMT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t dims[3] = {static_cast<uint64_t>(3 * d), static_cast<uint64_t>(seq), static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(3 * d) * 2, static_cast<uint64_t>(seq) * 3 * d * 2};
  CUtensorMap tq, tk, tv;
  const uint32_t box_q[3] = {64, attn::BQ, 1};
  const uint32_t box_k[3] = {64, attn::BKV / 2, 1};
  const uint32_t box_v[3] = {static_cast<uint32_t>(head_dim / 2), attn::BKV, 1};
  void* base = const_cast<void*>(qkv);
  if (!make_tmap(&tq, dt, 3, base, dims, strides, box_q, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tk, dt, 3, base, dims, strides, box_k, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tv, dt, 3, base, dims, strides, box_v,
                 head_dim == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  if (head_dim == 128)
    return fmt == FMT_F16 ? attn::launch_hd<128, FMT_F16>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s)
                          : attn::launch_hd<128, FMT_BF16>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s);
  return fmt == FMT_F16 ? attn::launch_hd<64, FMT_F16>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s)
                        : attn::launch_hd<64, FMT_BF16>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s);
}

}  // namespace jab
