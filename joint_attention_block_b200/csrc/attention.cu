// Joint bidirectional attention on the 5th-generation tensor cores.
//
// The Ideogram 4 DiT is single-stream: text and image tokens form one sequence
// through the same self-attention (Ideogram 4 deep dive, section 4-2; Ideogram 4.0
// announcement thread), so every query attends to every key with no mask:
//   O_h = softmax(q_h k_h^T / sqrt(hd)) v_h.
// A batch of prompts padded to one length passes a per-element key count; keys at or
// beyond it are left out of every row's softmax (padding sits at the end of each element).
//
// Two CTAs on two SMs (a cluster of 2) share 512 queries of one (batch, head) as two
// query tiles A and B of 256 rows; each CTA holds 128 rows of each tile.  The pair form of
// the MMA (tcgen05.mma.cta_group::2, M = 256) lets each CTA load only half of every
// key/value block:
//   S = Q K^T    N = 128 keys; CTA r loads keys [64 r, 64 r + 64) of the block
//   O += P V     N = hd;      CTA r loads value columns [r hd/2, (r + 1) hd/2) of the block,
//                             P (the A operand) is read from each CTA's own tensor memory,
// so a 4-stage key/value ring fits beside both query tiles.  Each tile owns 256 TMEM columns
// (S: 128 fp32 columns, O: hd columns); the tiles ping-pong so that the tensor core works on
// one tile while the other tile's softmax runs:
//     MMA issue order per key block j:  PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)
// The kernel is persistent: one CTA pair per SM pair walks the work items (batch element, head,
// 512 queries); the key/value ring and every barrier phase run on across items, the next item's
// S MMAs are issued as soon as its Q has landed, and its first P V waits only for this pair's
// epilogue of the previous item to have read O.
//   warp 0       TMA producer: per item, this CTA's rows of Q_A and Q_B (once the previous item's
//                S MMAs have read Q), then per key block its K and V halves, straight from the
//                fused qkv buffer [B, S, 3d]; every copy completes on the leader CTA's barriers.
//   warp 1       TMEM allocation (pair); in the leader, one lane issues the pair MMAs.
//   warps 2..5   softmax of tile A; warps 6..9 softmax of tile B.  Thread i owns query
//                row i of its tile (TMEM lane i), so the running max and sum are thread-local.
//                The whole row of S is read from TMEM at once; exp2 with the
//                log2(e)/sqrt(hd) scale folded in (packed fp32 pair arithmetic for the
//                scaling and the row sums).  P is written back over S in TMEM as 16-bit pairs.
//                The running max is only raised (and O rescaled in TMEM) when it grows
//                by more than 2^8; until then the stale max is used for both P and the
//                row sum, which leaves O / l unchanged and keeps P <= 256.  At the end
//                the same warps store O / l in the q/k/v format.
// e4m3 form (Q8, the W8A8 variant): Q and K come from separate e4m3 buffers [B, S, d] (one slab
// of hd bytes per row), S = Q K^T is issued as kind::f8f6f4 pair MMAs (K = 32 per instruction)
// and the two static scales of q and k multiply the softmax's log2(e)/sqrt(hd) factor; V, P and
// P V are as above.
#include "common.cuh"
#include "qk8.h"

namespace jab {
namespace attn {

constexpr int BQ = 128;   // rows of each query tile per CTA (a tile spans 256 rows of the pair)
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

// Q8: q and k as e4m3 bytes (one slab of hd bytes per row: 128-byte swizzle at hd = 128, 64-byte
// at hd = 64); otherwise 16-bit, in slabs of 64 values (128-byte rows, 128-byte swizzle).
template <int HD, bool Q8 = false>
struct Layout {
  static constexpr int Q_SLAB = Q8 ? 128 * HD : 128 * 128;
  static constexpr int Q_TILE = Q8 ? Q_SLAB : (HD / 64) * Q_SLAB;
  static constexpr int K_SLAB = Q8 ? 64 * HD : 64 * 128;
  static constexpr int K_BYTES = Q8 ? K_SLAB : (HD / 64) * K_SLAB;
  static constexpr int V_ROW = HD;  // bytes per key of this CTA's hd/2 value columns
  static constexpr int V_BYTES = BKV * V_ROW;
  static constexpr int OFF_Q = 0;  // [2] tiles
  static constexpr int OFF_K = OFF_Q + 2 * Q_TILE;
  static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * V_BYTES;
  static constexpr int NUM_BARS = 2 + 3 * STAGES + 8;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && V_BYTES % 1024 == 0,
                "swizzled tiles keep 1024-byte alignment");
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

// D[tmem] (+)= A * B^T for the CTA pair, kind::f8f6f4 with e4m3 A and B (q8 k8^T).
__device__ __forceinline__ void mma_e4m3_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// max(a, b, c) in one instruction (three-input form of max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Q8: tm_q / tm_k map the e4m3 q8 / k8 buffers ([B, S, d] bytes), qk_scale[0..1] their scales.
template <int HD, int F, bool Q8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out, int batch, int seq,
                     int n_heads, const int32_t* __restrict__ kv_len, const float* __restrict__ qk_scale,
                     const KernelGuard guard) {
  using L = Layout<HD, Q8>;
  constexpr bool kF16 = F == FMT_F16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;               // leader: both CTAs' Q rows of a work item landed
  uint64_t* q_empty = q_full + 1;        // every S MMA of a work item has read Q
  uint64_t* k_full = q_empty + 1;        // [STAGES] leader: both K halves of a block landed
  uint64_t* v_full = k_full + STAGES;    // [STAGES] leader: both V halves landed
  uint64_t* kv_empty = v_full + STAGES;  // [STAGES] both tiles' P V of the block are done
  uint64_t* s_full = kv_empty + STAGES;  // [2 tiles] S_t(j) ready (and P V_t(j-1) done)
  uint64_t* p_full = s_full + 2;         // [2 tiles] leader: both CTAs' P_t(j) written, O_t rescaled
  uint64_t* o_full = p_full + 2;         // both tiles' O of a work item final
  uint64_t* o_empty = o_full + 1;        // [2 tiles] leader: both CTAs' epilogue warps have read O_t
  uint64_t* drain_bar = o_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC + 4);

  const int warp = static_cast<int>(warp_id());
  const int lane = static_cast<int>(lane_id());
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  // Persistent: CTA pair p takes work items p, p + pairs, ...; item i = ((b * n_heads) + head) *
  // ntile + qt covers queries [512 qt, 512 qt + 512) of (b, head).
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;
  const int ntile = (seq + 4 * BQ - 1) / (4 * BQ);
  const int items = batch * n_heads * ntile;
  const int d = n_heads * HD;
  struct Item {
    int b, head, q0, nkv, nb;  // q0: this CTA's first row of tile A (tile t starts at q0 + 2 BQ t)
  };
  auto item = [&](int i) {
    Item it;
    const int qt = i % ntile;
    it.head = (i / ntile) % n_heads;
    it.b = i / (ntile * n_heads);
    it.q0 = qt * 4 * BQ + static_cast<int>(rank) * BQ;
    // keys of this batch element: all of them, or its key count (clamped to [1, seq])
    it.nkv = kv_len == nullptr ? seq : min(max(kv_len[it.b], 1), seq);
    it.nb = (it.nkv + BKV - 1) / BKV;
    return it;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 8);  // 4 softmax warps of the tile in each CTA
    }
    mbar_init(o_full, 1);
    mbar_init(&o_empty[0], 8);  // 4 epilogue warps of the tile in each CTA
    mbar_init(&o_empty[1], 8);
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

  if (warp == 0) {
    // ---------------- TMA producer: per work item this CTA's rows of Q_A and Q_B (once the
    // previous item's S MMAs have read Q), then its K and V halves of every key block, through
    // the key/value ring that runs on across items
    int issued = 0;    // key blocks issued, all items
    int q_issued = 0;  // work items whose Q load was issued
    int ui = 0;        // work items started
    bool ok = true;
    for (int i = pair; i < items && ok; i += pairs, ++ui) {
      const Item it = item(i);
      if (ui > 0 && !mbar_wait(q_empty, static_cast<uint32_t>(ui - 1) & 1u, guard, abort_flag,
                               where_code(ERR_TIMEOUT_ATTN_PRODUCER, rank, 0xFFFF))) {
        ok = false;
        break;
      }
      if (lane == 0) {
        if (leader) mbar_arrive_expect_tx(q_full, 2 * 2 * L::Q_TILE);
        const uint32_t qbar = mapa_shared(smem_u32(q_full), 0);
        for (int t = 0; t < 2; ++t) {
          if constexpr (Q8) {
            tma_load_3d_pair(sQ + t * L::Q_TILE, &tm_q, qbar, it.head * HD, it.q0 + 2 * BQ * t, it.b);
          } else {
            for (int c = 0; c < HD / 64; ++c)
              tma_load_3d_pair(sQ + t * L::Q_TILE + c * L::Q_SLAB, &tm_q, qbar, it.head * HD + 64 * c,
                               it.q0 + 2 * BQ * t, it.b);
          }
        }
      }
      __syncwarp();
      ++q_issued;
      for (int j = 0; j < it.nb; ++j) {
        const int st = issued % STAGES;
        const uint32_t rnd = static_cast<uint32_t>(issued / STAGES);
        if (!mbar_wait(&kv_empty[st], (rnd & 1u) ^ 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_ATTN_PRODUCER, rank, issued))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          if (leader) {
            mbar_arrive_expect_tx(&k_full[st], 2 * L::K_BYTES);
            mbar_arrive_expect_tx(&v_full[st], 2 * L::V_BYTES);
          }
          const uint32_t kbar = mapa_shared(smem_u32(&k_full[st]), 0);
          const uint32_t vbar = mapa_shared(smem_u32(&v_full[st]), 0);
          if constexpr (Q8) {
            tma_load_3d_pair(sK + st * L::K_BYTES, &tm_k, kbar, it.head * HD, j * BKV + 64 * static_cast<int>(rank),
                             it.b);
          } else {
            for (int c = 0; c < HD / 64; ++c)
              tma_load_3d_pair(sK + st * L::K_BYTES + c * L::K_SLAB, &tm_k, kbar, d + it.head * HD + 64 * c,
                               j * BKV + 64 * static_cast<int>(rank), it.b);
          }
          tma_load_3d_pair(sV + st * L::V_BYTES, &tm_v, vbar,
                           2 * d + it.head * HD + static_cast<int>(rank) * (HD / 2), j * BKV, it.b);
        }
        __syncwarp();
        ++issued;
      }
    }
    // Never leave with copies in flight: the leader's barriers count both CTAs' copies, and
    // the peer is held by the final cluster barrier until the leader has drained.  At most one
    // Q load is outstanding (each waits for the previous item's S MMAs).
    if (leader) {
      if (q_issued > 0)
        mbar_wait(q_full, static_cast<uint32_t>(q_issued - 1) & 1u, guard, abort_flag,
                  where_code(ERR_TIMEOUT_ATTN_DRAIN, rank, 0), true);
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
      // kind::f16 for 16-bit q, k; kind::f8f6f4 (type code 0: e4m3) for Q8
      constexpr uint32_t idesc_s = idesc_f16kind(2 * BQ, BKV, Q8 ? true : kF16, false, false);
      constexpr uint32_t idesc_o = idesc_f16kind(2 * BQ, HD, kF16, false, true);
      // g: key block index over all work items (the ring slot and the barrier phases); j: the
      // block within the item
      auto issue_s = [&](int t, int g) {  // S_t = Q_t K_g^T into columns [256 t, 256 t + 128)
        const uint32_t qbase = smem_u32(sQ + t * L::Q_TILE);
        const uint32_t kbase = smem_u32(sK + (g % STAGES) * L::K_BYTES);
        if constexpr (Q8) {
#pragma unroll
          for (int kk = 0; kk < HD / 32; ++kk) {  // 32 e4m3 values (32 bytes) per MMA
            const uint64_t qd = HD == 128 ? smem_desc_sw128(qbase + 32 * kk, 16, 1024) : smem_desc_sw64(qbase + 32 * kk, 16, 512);
            const uint64_t kd = HD == 128 ? smem_desc_sw128(kbase + 32 * kk, 16, 1024) : smem_desc_sw64(kbase + 32 * kk, 16, 512);
            mma_e4m3_ss_pair(tmem + 256 * t, qd, kd, idesc_s, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t oq = (kk >> 2) * L::Q_SLAB + (kk & 3) * 32;
            const uint32_t ok_ = (kk >> 2) * L::K_SLAB + (kk & 3) * 32;
            mma_f16kind_ss_pair(tmem + 256 * t, smem_desc_sw128(qbase + oq, 16, 1024),
                                smem_desc_sw128(kbase + ok_, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit_pair(&s_full[t], 0x3);
      };
      auto issue_pv = [&](int t, int g, int j) {  // O_t += P_t V_g, P from TMEM (columns [256 t, 256 t + 64))
        const uint32_t vbase = smem_u32(sV + (g % STAGES) * L::V_BYTES);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint32_t a = vbase + kk * 16 * L::V_ROW;
          const uint64_t bd = HD == 128 ? smem_desc_sw128(a, 16, 8 * L::V_ROW) : smem_desc_sw64(a, 16, 8 * L::V_ROW);
          mma_f16kind_ts_pair(tmem + 256 * t + 128, tmem + 256 * t + 8 * kk, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = true;
      int gb = 0;  // key blocks of the items before this one
      int ui = 0;
      for (int i = pair; i < items && ok; i += pairs, ++ui) {
        const Item it = item(i);
        const int nb = it.nb;
        // S_A(0), S_B(0) overwrite S (and P) of the previous item only after its P V MMAs,
        // issued before them, have read P
        ok = mbar_wait(q_full, static_cast<uint32_t>(ui) & 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_ATTN_MMA, rank, 0)) &&
             mbar_wait(&k_full[gb % STAGES], static_cast<uint32_t>(gb / STAGES) & 1u, guard, abort_flag,
                       where_code(ERR_TIMEOUT_ATTN_MMA, rank, gb));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_s(0, gb);
          issue_s(1, gb);
          if (nb == 1) mma_commit_pair(q_empty, 0x3);  // the item's last S MMAs are issued: Q free after them
        }
        __syncwarp();
        for (int j = 0; j < nb && ok; ++j) {
          const int g = gb + j;
          const int st = g % STAGES;
          const uint32_t par = static_cast<uint32_t>(g) & 1u;
          const bool next = j + 1 < nb;
          // the first P V of an item overwrites O_t: both CTAs' epilogues of the previous item
          // must have read it
          ok = mbar_wait(&v_full[st], static_cast<uint32_t>(g / STAGES) & 1u, guard, abort_flag,
                         where_code(ERR_TIMEOUT_ATTN_MMA, 1, g)) &&
               mbar_wait(&p_full[0], par, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_MMA, 2, g)) &&
               (!next || mbar_wait(&k_full[(g + 1) % STAGES], static_cast<uint32_t>((g + 1) / STAGES) & 1u, guard,
                                   abort_flag, where_code(ERR_TIMEOUT_ATTN_MMA, 3, g))) &&
               (j > 0 || ui == 0 ||
                mbar_wait(&o_empty[0], static_cast<uint32_t>(ui - 1) & 1u, guard, abort_flag,
                          where_code(ERR_TIMEOUT_ATTN_MMA, 5, g)));
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            issue_pv(0, g, j);
            if (next) issue_s(0, g + 1);  // overwrites P_A only after P V_A has read it (in-order issue)
          }
          __syncwarp();
          ok = mbar_wait(&p_full[1], par, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_MMA, 4, g)) &&
               (j > 0 || ui == 0 ||
                mbar_wait(&o_empty[1], static_cast<uint32_t>(ui - 1) & 1u, guard, abort_flag,
                          where_code(ERR_TIMEOUT_ATTN_MMA, 6, g)));
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            issue_pv(1, g, j);
            mma_commit_pair(&kv_empty[st], 0x3);  // K_g and V_g fully consumed by both tiles
            if (next) {
              issue_s(1, g + 1);
              if (j + 2 == nb) mma_commit_pair(q_empty, 0x3);  // the item's last S MMAs are issued
            }
          }
          __syncwarp();
        }
        if (ok && lane == 0) mma_commit_pair(o_full, 0x3);  // this item's O final
        __syncwarp();
        gb += nb;
      }
      if (lane == 0) mma_commit_pair(drain_bar, 0x3);  // all MMAs retired before either CTA frees TMEM
      __syncwarp();
    }
    mbar_wait(drain_bar, 0u, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_DRAIN, rank, 1), true);
  } else {
    // ---------------- softmax: warps 2..5 -> tile A, 6..9 -> tile B; thread owns query row
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_col = tmem + lane_off + 256 * t;
    const uint32_t o_col = s_col + 128;
    // log2(e) / sqrt(hd), the same fp32 quotient as dividing by the fp32 square root of hd
    // (Q8: times the two e4m3 scales, S being accumulated from the codes)
    constexpr float c_log2_16 = 1.4426950408889634f / (HD == 128 ? 11.313708498984761f : 8.0f);
    const float c_log2 = Q8 ? c_log2_16 * (qk_scale[0] * qk_scale[1]) : c_log2_16;
    bool ok = true;
    uint32_t sph = 0u;  // phase parity of s_full[t]: one phase per key block, all items
    for (int ui = 0; pair + ui * pairs < items && ok; ++ui) {
    int nkv, nb;
    {
      const Item it = item(pair + ui * pairs);
      nkv = it.nkv;
      nb = it.nb;
    }
    float m_used = -INFINITY;
    float l = 0.f;
    for (int j = 0; j < nb; ++j) {
      if (!mbar_wait(&s_full[t], sph, guard, abort_flag, where_code(ERR_TIMEOUT_ATTN_SOFTMAX, rank * 2 + t, j))) {
        ok = false;
        break;
      }
      sph ^= 1u;
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
        alpha = ex2_approx(m_used - mx);  // 0 on the first block
        m_used = mx;
        rescale = true;
      }
      // exponentiate, sum, and write P_t(j) as 16-bit pairs over the first 64 columns of S_t
      // (the A operand of the PV MMA)
      float2 ps[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 c2 = make_float2(c_log2, c_log2);
      const float2 nm2 = make_float2(-m_used, -m_used);
#pragma unroll
      for (int h = 0; h < 4; ++h) {  // four 32-key chunks: 16 packed columns each
        uint32_t pk[16];
#pragma unroll
        for (int k2 = 0; k2 < 32; k2 += 2) {
          const int k = 32 * h + k2;
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
        tmem_st16(s_col + 16 * h, pk);
      }
      const float2 ps01 = add2(ps[0], ps[1]), ps23 = add2(ps[2], ps[3]);
      const float2 ps03 = add2(ps01, ps23);
      const float sum = ps03.x + ps03.y;
      // O_t is up to date here: PV_t(j-1) was issued before S_t(j) and s_full covers it.
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
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
      if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&p_full[t]), 0));
    }
    if (!ok) break;
    if (!mbar_wait(o_full, static_cast<uint32_t>(ui) & 1u, guard, abort_flag,
                   where_code(ERR_TIMEOUT_ATTN_SOFTMAX, 4 + rank, t))) {
      ok = false;
      break;
    }
    {
      tc_fence_after();
      const Item it = item(pair + ui * pairs);
      const float inv_l = 1.f / l;
      const int row = it.q0 + 2 * BQ * t + r;
      uint16_t* dst = out + (static_cast<size_t>(it.b) * seq + row) * d + it.head * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(o_col + 32 * c, raw);
        tmem_ld_wait();
        if (row < seq) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float o[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] = __uint_as_float(raw[8 * q + k]) * inv_l;
            store8<F>(dst + 32 * c, q, o);
          }
        }
      }
    }
    // O_t read: the next item's first P V may overwrite it
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&o_empty[t]), 0));
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

template <int HD, int F, bool Q8 = false>
cudaError_t launch_hd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* out, int batch,
                      int seq, int n_heads, const int32_t* kv_len, const KernelGuard& g, cudaStream_t s,
                      const float* qk_scale = nullptr) {
  using L = Layout<HD, Q8>;
  cudaError_t e =
      cudaFuncSetAttribute(attention_kernel<HD, F, Q8>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  // persistent: one CTA pair per SM pair at most, each walking work items (b, head, 512 queries)
  const long long items = static_cast<long long>(batch) * n_heads * ((seq + 4 * BQ - 1) / (4 * BQ));
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  const long long pairs = items < sms / 2 ? items : sms / 2;
  if (items >= (1ll << 31) || pairs < 1) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(2 * pairs), 1, 1);
  return launch_pdl(attention_kernel<HD, F, Q8>, grid, dim3(THREADS), L::SMEM, s, tq, tk, tv,
                    static_cast<uint16_t*>(out), batch, seq, n_heads, kv_len, qk_scale, g);
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


cudaError_t launch_attention_q8(const uint8_t* q8, const uint8_t* k8, const float* scale, const void* qkv, void* out,
                                int fmt, int batch, int seq, int n_heads, int head_dim, const int32_t* kv_len,
                                const KernelGuard& g, cudaStream_t s) {
  if (batch <= 0 || seq <= 0) return cudaSuccess;
  if (fmt != FMT_BF16 && fmt != FMT_F16) return cudaErrorInvalidValue;
  if (head_dim != 64 && head_dim != 128) return cudaErrorInvalidValue;
  if (q8 == nullptr || k8 == nullptr || scale == nullptr) return cudaErrorInvalidValue;
  const int d = n_heads * head_dim;
  const CUtensorMapDataType dt = fmt == FMT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // e4m3 q and k: [B, S, d] bytes, one box of hd bytes per row (x = head * hd, a multiple of 64)
  const uint64_t dims8[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(seq), static_cast<uint64_t>(batch)};
  const uint64_t strides8[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(seq) * d};
  const uint64_t dims[3] = {static_cast<uint64_t>(3 * d), static_cast<uint64_t>(seq), static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(3 * d) * 2, static_cast<uint64_t>(seq) * 3 * d * 2};
  CUtensorMap tq, tk, tv;
  const uint32_t box_q[3] = {static_cast<uint32_t>(head_dim), attn::BQ, 1};
  const uint32_t box_k[3] = {static_cast<uint32_t>(head_dim), attn::BKV / 2, 1};
  const uint32_t box_v[3] = {static_cast<uint32_t>(head_dim / 2), attn::BKV, 1};
  const CUtensorMapSwizzle swz = head_dim == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(q8), dims8, strides8, box_q, swz) ||
      !make_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(k8), dims8, strides8, box_k, swz) ||
      !make_tmap(&tv, dt, 3, const_cast<void*>(qkv), dims, strides, box_v, swz))
    return cudaErrorInvalidValue;
  if (head_dim == 128)
    return fmt == FMT_F16 ? attn::launch_hd<128, FMT_F16, true>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s, scale)
                          : attn::launch_hd<128, FMT_BF16, true>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s, scale);
  return fmt == FMT_F16 ? attn::launch_hd<64, FMT_F16, true>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s, scale)
                        : attn::launch_hd<64, FMT_BF16, true>(tq, tk, tv, out, batch, seq, n_heads, kv_len, g, s, scale);
}
}  // namespace jab
