// The C ABI: argument validation, workspace carving and the composition of the
// block forward, the conditioning projection and the CFG/Euler step from the
// kernels in the other translation units.
#include <cudaTypedefs.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "jab_dit.h"
#include "internal.h"
#include "qk8.h"

namespace jab {

// ------------------------------------------------------------------ device error word

// One word per device: the first device-side error recorded since the last poll.
__device__ uint32_t g_device_error;

static std::atomic<uint64_t> g_timeout_ns{2000ull * 1000ull * 1000ull};
static std::mutex g_mu;
static uint32_t* g_err_ptr[64] = {nullptr};

cudaError_t current_guard(KernelGuard* g) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return e;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
  }
  g->err = g_err_ptr[dev];
  g->timeout_ns = g_timeout_ns.load();
  return cudaSuccess;
}

// ------------------------------------------------------------------ TMA descriptors

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  cuuint64_t gdim[3], gstr[2];
  cuuint32_t bdim[3];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gstr[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank), base, gdim, gstr, bdim, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launch instrumentation

// When enabled, every launch of the three calls whose tag is in the mask is bracketed by
// CUDA events on its stream (tag = which kernel), so a caller can read per-kernel device
// time of the very launches it timed.  A mark starts the kernel launched after it and ends
// the one before it: an END event is recorded only where a bracketed kernel is followed by
// one that is not.  Off by default; events are created once, at enable time.
struct ProfState {
  bool on = false;
  int cap = 0;
  int n = 0;
  uint32_t mask = 0xFFFFFFFFu;
  bool open = false;  // the last recorded event starts a bracketed kernel
  cudaEvent_t* ev = nullptr;
  int* tag = nullptr;
};
static ProfState g_prof;
static std::mutex g_prof_mu;

void prof_mark(cudaStream_t s, int tag) {
  if (!g_prof.on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  const bool want = tag != DIT_KERNEL_END && tag < 32 && ((g_prof.mask >> tag) & 1u) != 0u;
  if (!want && !g_prof.open) return;  // nothing to end, nothing to start
  if (g_prof.n >= g_prof.cap) return;
  cudaEventRecord(g_prof.ev[g_prof.n], s);
  g_prof.tag[g_prof.n] = want ? tag : DIT_KERNEL_END;
  ++g_prof.n;
  g_prof.open = want;
}

}  // namespace jab

using namespace jab;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

std::atomic<int> g_last_cuda_error{0};

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return DIT_OK;
  g_last_cuda_error.store(static_cast<int>(e));
  return DIT_ERR_CUDA;
}

// A launch error is reported once by the next cudaGetLastError() of the thread; clear any that an
// earlier, unrelated call left behind so that it is not reported as this call's failure.
void clear_stale_error() { (void)cudaGetLastError(); }

int check_config(const dit_block_config* c) {
  if (c == nullptr) return DIT_ERR_INVALID_ARG;
  if (c->n_heads <= 0 || c->head_dim <= 0 || c->d_model != c->n_heads * c->head_dim) return DIT_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return DIT_ERR_UNSUPPORTED;
  if (c->d_model % 256 != 0 || c->d_mlp <= 0 || c->d_mlp % 256 != 0) return DIT_ERR_UNSUPPORTED;
  if (c->d_model > 8192) return DIT_ERR_UNSUPPORTED;  // the QK-norm kernel: one CTA of d/16 <= 512 threads per token
  if (c->rope_sections[0] < 0 || c->rope_sections[1] < 0 || c->rope_sections[2] < 0) return DIT_ERR_INVALID_ARG;
  if (c->rope_sections[0] + c->rope_sections[1] + c->rope_sections[2] != c->head_dim / 2) return DIT_ERR_INVALID_ARG;
  if (!(c->rope_theta > 0.f) || !(c->eps >= 0.f)) return DIT_ERR_INVALID_ARG;
  return DIT_OK;
}

// Internal activations: h, qkv, o, u in f16 (every one is bounded: post-norm,
// softmax-weighted or a GEMM of bounded inputs); the residual x1 in fp32.
// The rotary tables hold one [S, hd/2] pair per batch element (padded batches position each
// element on its own; otherwise only the first is used) and kv_len the per-element key counts.
struct BlockWorkspace {
  int32_t* kv_len;
  uint16_t* h;
  uint16_t* qkv;
  uint16_t* o;
  float* x1;
  uint16_t* u;
  float* sa;  // per-token e4m3 scales of the W8A8 variant (its e4m3 codes reuse h)
  float* qk8_scale;  // W8A8: the static e4m3 scales of q and k (their codes reuse h after the QKV GEMM)
  size_t bytes;
};

BlockWorkspace carve_block(const dit_block_config* c, int batch, int seq, void* base) {
  BlockWorkspace w{};
  const size_t M = static_cast<size_t>(batch) * seq;
  const size_t d = c->d_model, F = c->d_mlp;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t o_kv = take(static_cast<size_t>(batch) * 4);
  const size_t o_h = take(M * d * 2), o_qkv = take(M * 3 * d * 2), o_o = take(M * d * 2), o_x1 = take(M * d * 4);
  const size_t o_u = take(M * F * 2), o_sa = take(M * 4), o_qs = take(2 * 4);
  w.bytes = off;
  if (base != nullptr) {
    uint8_t* b = static_cast<uint8_t*>(base);
    w.kv_len = reinterpret_cast<int32_t*>(b + o_kv);
    w.h = reinterpret_cast<uint16_t*>(b + o_h);
    w.qkv = reinterpret_cast<uint16_t*>(b + o_qkv);
    w.o = reinterpret_cast<uint16_t*>(b + o_o);
    w.x1 = reinterpret_cast<float*>(b + o_x1);
    w.u = reinterpret_cast<uint16_t*>(b + o_u);
    w.sa = reinterpret_cast<float*>(b + o_sa);
    w.qk8_scale = reinterpret_cast<float*>(b + o_qs);
  }
  return w;
}

bool shape_ok(int batch, int n_text, int grid_h, int grid_w) {
  if (batch <= 0 || n_text < 0 || grid_h < 0 || grid_w < 0) return false;
  const int64_t S = static_cast<int64_t>(n_text) + static_cast<int64_t>(grid_h) * grid_w;
  return S > 0 && S * batch < (1ll << 31) / 16;
}

}  // namespace

extern "C" {

int dit_abi_version(void) { return 2; }

int dit_last_cuda_error(void) { return g_last_cuda_error.load(); }

int dit_profile_enable(int max_marks) { return dit_profile_enable_tags(max_marks, 0xFFFFFFFFu); }

int dit_profile_enable_tags(int max_marks, uint32_t tag_mask) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (max_marks <= 0 || tag_mask == 0u) return DIT_ERR_INVALID_ARG;
  if (g_prof.cap < max_marks) {
    for (int i = 0; i < g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
    delete[] g_prof.ev;
    delete[] g_prof.tag;
    g_prof.ev = new cudaEvent_t[max_marks];
    g_prof.tag = new int[max_marks];
    for (int i = 0; i < max_marks; ++i)
      if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) {
        g_prof.cap = i;
        return DIT_ERR_CUDA;
      }
    g_prof.cap = max_marks;
  }
  g_prof.n = 0;
  g_prof.mask = tag_mask;
  g_prof.open = false;
  g_prof.on = true;
  return DIT_OK;
}

int dit_profile_disable(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof.on = false;
  return DIT_OK;
}

int dit_profile_read(int* tags, float* ms, int max_records) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int out = 0;
  for (int i = 0; i + 1 < g_prof.n && out < max_records; ++i) {
    if (g_prof.tag[i] == DIT_KERNEL_END) continue;
    float t = 0.f;
    if (cudaEventSynchronize(g_prof.ev[i + 1]) != cudaSuccess) return -DIT_ERR_CUDA;
    if (cudaEventElapsedTime(&t, g_prof.ev[i], g_prof.ev[i + 1]) != cudaSuccess) return -DIT_ERR_CUDA;
    tags[out] = g_prof.tag[i];
    ms[out] = t;
    ++out;
  }
  g_prof.n = 0;
  return out;
}

const char* dit_status_str(int s) {
  switch (s) {
    case DIT_OK: return "ok";
    case DIT_ERR_INVALID_ARG: return "invalid argument";
    case DIT_ERR_UNSUPPORTED: return "unsupported size";
    case DIT_ERR_WORKSPACE: return "workspace missing or too small";
    case DIT_ERR_CUDA: return "CUDA error";
    case DIT_ERR_TIMEOUT: return "device-side bounded wait timed out";
    case DIT_ERR_DEVICE: return "device-side error";
    default: return "unknown status";
  }
}

int dit_set_wait_timeout_ms(uint32_t ms) {
  if (ms == 0) return DIT_ERR_INVALID_ARG;
  g_timeout_ns.store(static_cast<uint64_t>(ms) * 1000000ull);
  return DIT_OK;
}

static std::atomic<uint32_t> g_last_device_error{0};

uint32_t dit_last_device_error(void) { return g_last_device_error.load(); }

int dit_poll_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return DIT_ERR_CUDA;
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return DIT_ERR_CUDA;
  if (v == 0) return DIT_OK;
  g_last_device_error.store(v);
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return DIT_ERR_CUDA;
  return (v & 0xF00u) == 0x100u ? DIT_ERR_TIMEOUT : DIT_ERR_DEVICE;
}

int dit_wait_selftest(void* stream) {
  clear_stale_error();
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  return from_cuda(launch_wait_selftest(g, as_stream(stream)));
}

int dit_e4m3_to_bf16(const uint8_t* codes, void* out, int64_t n, void* stream) {
  clear_stale_error();
  if (n < 0 || (n > 0 && (codes == nullptr || out == nullptr))) return DIT_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(out)) return DIT_ERR_INVALID_ARG;
  return from_cuda(launch_e4m3_to_bf16(codes, static_cast<uint16_t*>(out), n, as_stream(stream)));
}

int dit_rmsnorm_rows(const void* x, int x_fmt, const void* g, void* y, int y_fmt, int64_t rows, int64_t cols,
                     float eps, void* stream) {
  clear_stale_error();
  if (rows < 0 || cols <= 0 || cols % 8 != 0 || rows > (1ll << 31) - 1) return DIT_ERR_INVALID_ARG;
  if ((x_fmt != FMT_BF16 && x_fmt != FMT_F32) || (y_fmt != FMT_BF16 && y_fmt != FMT_F16)) return DIT_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || g == nullptr || y == nullptr)) return DIT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(g) || !aligned16(y)) return DIT_ERR_INVALID_ARG;
  if (x == y && x_fmt != y_fmt) return DIT_ERR_INVALID_ARG;
  prof_mark(as_stream(stream), DIT_KERNEL_RMSNORM);
  const cudaError_t e =
      launch_rmsnorm(x, x_fmt, static_cast<const uint16_t*>(g), y, y_fmt, rows, cols, eps, as_stream(stream));
  prof_mark(as_stream(stream), DIT_KERNEL_END);
  return from_cuda(e);
}

int euler_cfg_step(float* x, const void* v_cond, const void* v_uncond, int64_t n, float guidance, float dt,
                   void* stream) {
  clear_stale_error();
  if (n < 0 || (n > 0 && (x == nullptr || v_cond == nullptr || v_uncond == nullptr))) return DIT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(v_cond) || !aligned16(v_uncond)) return DIT_ERR_INVALID_ARG;
  prof_mark(as_stream(stream), DIT_KERNEL_EULER_CFG);
  const cudaError_t e = launch_euler_cfg(x, static_cast<const uint16_t*>(v_cond),
                                         static_cast<const uint16_t*>(v_uncond), n, guidance, dt, as_stream(stream));
  prof_mark(as_stream(stream), DIT_KERNEL_END);
  return from_cuda(e);
}

int dit_mrope_positions(int n_text, int grid_h, int grid_w, int t_img, int32_t* pos_out, void* stream) {
  clear_stale_error();
  if (!shape_ok(1, n_text, grid_h, grid_w) || pos_out == nullptr) return DIT_ERR_INVALID_ARG;
  if (t_img < 0) t_img = n_text;
  return from_cuda(launch_positions(n_text, grid_h, grid_w, t_img, pos_out, as_stream(stream)));
}

int dit_gemm_w8a16(const void* a, int a_fmt, const uint8_t* w8, const float* scale, void* y, int y_fmt,
                   const void* residual, int res_fmt, int M, int N, int K, int act, int gelu_tanh, void* stream) {
  clear_stale_error();
  if (M < 0 || N <= 0 || K <= 0) return DIT_ERR_INVALID_ARG;
  if (N % 32 != 0 || K % 16 != 0) return DIT_ERR_UNSUPPORTED;
  if ((a_fmt != FMT_BF16 && a_fmt != FMT_F16) || y_fmt < FMT_BF16 || y_fmt > FMT_F32) return DIT_ERR_INVALID_ARG;
  if (act < 0 || act > 1) return DIT_ERR_INVALID_ARG;
  if (residual != nullptr && (res_fmt < FMT_BF16 || res_fmt > FMT_F32)) return DIT_ERR_INVALID_ARG;
  if (M == 0) return DIT_OK;
  if (a == nullptr || w8 == nullptr || scale == nullptr || y == nullptr) return DIT_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w8) || !aligned16(y) || !aligned16(residual)) return DIT_ERR_INVALID_ARG;
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  GemmArgs args{a, a_fmt, w8, scale, y, y_fmt, residual, res_fmt, M, N, K, act, gelu_tanh};
  return from_cuda(launch_gemm_w8a16(args, g, as_stream(stream)));
}

int dit_qknorm_mrope(void* qkv, int fmt, int batch, int n_text, int grid_h, int grid_w, int t_img, const int32_t* pos,
                     const dit_block_config* cfg, const void* g_q, const void* g_k, void* workspace, size_t ws_bytes,
                     void* stream) {
  clear_stale_error();
  int st = check_config(cfg);
  if (st != DIT_OK) return st;
  if (!shape_ok(batch, n_text, grid_h, grid_w) || qkv == nullptr || g_q == nullptr || g_k == nullptr)
    return DIT_ERR_INVALID_ARG;
  if (fmt != FMT_BF16 && fmt != FMT_F16) return DIT_ERR_INVALID_ARG;
  const int S = n_text + grid_h * grid_w;
  (void)workspace;  // the rotary angles are computed in the kernel; no scratch is needed
  (void)ws_bytes;
  cudaStream_t s = as_stream(stream);
  prof_mark(s, DIT_KERNEL_QKNORM_MROPE);
  cudaError_t e = launch_qknorm_mrope(qkv, fmt, batch, S, cfg->n_heads, cfg->head_dim, n_text, grid_w,
                                      grid_h * grid_w, t_img, pos, nullptr, nullptr, cfg->rope_sections,
                                      cfg->rope_theta, static_cast<const uint16_t*>(g_q),
                                      static_cast<const uint16_t*>(g_k), cfg->eps, s);
  prof_mark(s, DIT_KERNEL_END);
  return from_cuda(e);
}

int dit_qknorm_mrope_e4m3(const void* qkv, int fmt, int batch, int n_text, int grid_h, int grid_w, int t_img,
                          const int32_t* pos, const dit_block_config* cfg, const void* g_q, const void* g_k,
                          uint8_t* q8, uint8_t* k8, float* scale, void* stream) {
  clear_stale_error();
  int st = check_config(cfg);
  if (st != DIT_OK) return st;
  if (!shape_ok(batch, n_text, grid_h, grid_w) || qkv == nullptr || g_q == nullptr || g_k == nullptr ||
      q8 == nullptr || k8 == nullptr || scale == nullptr)
    return DIT_ERR_INVALID_ARG;
  if (fmt != FMT_BF16 && fmt != FMT_F16) return DIT_ERR_INVALID_ARG;
  if (!aligned16(qkv) || !aligned16(q8) || !aligned16(k8)) return DIT_ERR_INVALID_ARG;
  const int S = n_text + grid_h * grid_w;
  cudaStream_t s = as_stream(stream);
  const QK8Out o8{q8, k8, scale};
  prof_mark(s, DIT_KERNEL_QKNORM_MROPE);
  cudaError_t e = launch_qknorm_mrope_e4m3(qkv, fmt, batch, S, cfg->n_heads, cfg->head_dim, n_text, grid_w,
                                           grid_h * grid_w, t_img, pos, nullptr, nullptr, cfg->rope_sections,
                                           cfg->rope_theta, static_cast<const uint16_t*>(g_q),
                                           static_cast<const uint16_t*>(g_k), cfg->eps, o8, s);
  prof_mark(s, DIT_KERNEL_END);
  return from_cuda(e);
}

int dit_joint_attention_e4m3(const uint8_t* q8, const uint8_t* k8, const float* scale, const void* qkv, void* out,
                             int fmt, int batch, int seq, int n_heads, int head_dim, void* stream) {
  clear_stale_error();
  if (batch <= 0 || seq <= 0 || n_heads <= 0 || qkv == nullptr || out == nullptr || q8 == nullptr ||
      k8 == nullptr || scale == nullptr)
    return DIT_ERR_INVALID_ARG;
  if (fmt != FMT_BF16 && fmt != FMT_F16) return DIT_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(q8) || !aligned16(k8)) return DIT_ERR_INVALID_ARG;
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  return from_cuda(
      launch_attention_q8(q8, k8, scale, qkv, out, fmt, batch, seq, n_heads, head_dim, nullptr, g, as_stream(stream)));
}

int dit_joint_attention(const void* qkv, void* out, int fmt, int batch, int seq, int n_heads, int head_dim,
                        void* stream) {
  clear_stale_error();
  if (batch <= 0 || seq <= 0 || n_heads <= 0 || qkv == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if (fmt != FMT_BF16 && fmt != FMT_F16) return DIT_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(qkv) || !aligned16(out)) return DIT_ERR_INVALID_ARG;
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  return from_cuda(launch_attention(qkv, out, fmt, batch, seq, n_heads, head_dim, nullptr, g, as_stream(stream)));
}

size_t dit_block_workspace_bytes(const dit_block_config* cfg, int batch, int n_text, int grid_h, int grid_w) {
  if (check_config(cfg) != DIT_OK || !shape_ok(batch, n_text, grid_h, grid_w)) return 0;
  return carve_block(cfg, batch, n_text + grid_h * grid_w, nullptr).bytes;
}

}  // extern "C"

namespace {

// The block forward behind dit_block_forward (text_lens == nullptr) and dit_block_forward_padded.
int block_forward(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in, void* x_out, int batch,
                  int n_text, int grid_h, int grid_w, int t_img, const int32_t* pos, const int32_t* text_lens,
                  void* workspace, size_t ws_bytes, void* stream, bool w8a8 = false) {
  clear_stale_error();
  int st = check_config(cfg);
  if (st != DIT_OK) return st;
  if (w == nullptr || x_in == nullptr || x_out == nullptr || x_in == x_out) return DIT_ERR_INVALID_ARG;
  if (!shape_ok(batch, n_text, grid_h, grid_w)) return DIT_ERR_INVALID_ARG;
  const void* ptrs[] = {w->w_qkv, w->w_o, w->w_up, w->w_down, w->s_qkv, w->s_o, w->s_up, w->s_down, w->g_norm1,
                        w->g_norm2, w->g_q, w->g_k};
  for (const void* p : ptrs)
    if (p == nullptr) return DIT_ERR_INVALID_ARG;
  if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(w->w_qkv) || !aligned16(w->w_o) || !aligned16(w->w_up) ||
      !aligned16(w->w_down) || !aligned16(w->g_norm1) || !aligned16(w->g_norm2) || !aligned16(w->g_q) ||
      !aligned16(w->g_k))
    return DIT_ERR_INVALID_ARG;
  const int S = n_text + grid_h * grid_w;
  BlockWorkspace ws = carve_block(cfg, batch, S, nullptr);
  if (workspace == nullptr || ws_bytes < ws.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return DIT_ERR_WORKSPACE;
  ws = carve_block(cfg, batch, S, workspace);
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const int M = batch * S, d = cfg->d_model, F = cfg->d_mlp;
  const uint16_t* x = static_cast<const uint16_t*>(x_in);
  uint16_t* y = static_cast<uint16_t*>(x_out);

#define JAB_TRY(expr)                         \
  do {                                        \
    const cudaError_t jab_e = (expr);         \
    if (jab_e != cudaSuccess) return from_cuda(jab_e); \
  } while (0)
  const bool padded = text_lens != nullptr;
  const uint16_t* g1 = static_cast<const uint16_t*>(w->g_norm1);
  const uint16_t* g2 = static_cast<const uint16_t*>(w->g_norm2);
  uint8_t* h8 = reinterpret_cast<uint8_t*>(ws.h);  // e4m3 codes of the W8A8 variant
  prof_mark(s, DIT_KERNEL_RMSNORM);
  if (w8a8)
    JAB_TRY(launch_rmsnorm_e4m3(x, FMT_BF16, g1, h8, ws.sa, M, d, cfg->eps, s));
  else
    JAB_TRY(launch_rmsnorm(x, FMT_BF16, g1, ws.h, FMT_F16, M, d, cfg->eps, s));
  prof_mark(s, DIT_KERNEL_GEMM_QKV);
  if (w8a8)
    JAB_TRY(launch_gemm_w8a8(GemmArgs8{h8, ws.sa, w->w_qkv, w->s_qkv, ws.qkv, FMT_F16, M, 3 * d, d, 0, 0}, g, s));
  else
    JAB_TRY(launch_gemm_w8a16(
        GemmArgs{ws.h, FMT_F16, w->w_qkv, w->s_qkv, ws.qkv, FMT_F16, nullptr, -1, M, 3 * d, d, 0, 0}, g, s));
  prof_mark(s, DIT_KERNEL_QKNORM_MROPE);
  // W8A8: q and k as e4m3 codes over h (free once the QKV GEMM has read it): q8 = h[0, M d),
  // k8 = h[M d, 2 M d) bytes
  const QK8Out o8{h8, h8 + static_cast<size_t>(M) * d, ws.qk8_scale};
  if (w8a8)
    JAB_TRY(launch_qknorm_mrope_e4m3(ws.qkv, FMT_F16, batch, S, cfg->n_heads, cfg->head_dim, n_text, grid_w,
                                     grid_h * grid_w, t_img, pos, text_lens, padded ? ws.kv_len : nullptr,
                                     cfg->rope_sections, cfg->rope_theta, static_cast<const uint16_t*>(w->g_q),
                                     static_cast<const uint16_t*>(w->g_k), cfg->eps, o8, s));
  else
    JAB_TRY(launch_qknorm_mrope(ws.qkv, FMT_F16, batch, S, cfg->n_heads, cfg->head_dim, n_text, grid_w,
                                grid_h * grid_w, t_img, pos, text_lens, padded ? ws.kv_len : nullptr,
                                cfg->rope_sections, cfg->rope_theta, static_cast<const uint16_t*>(w->g_q),
                                static_cast<const uint16_t*>(w->g_k), cfg->eps, s));
  prof_mark(s, DIT_KERNEL_ATTENTION);
  if (w8a8)
    JAB_TRY(launch_attention_q8(o8.q8, o8.k8, o8.scale, ws.qkv, ws.o, FMT_F16, batch, S, cfg->n_heads, cfg->head_dim,
                                padded ? ws.kv_len : nullptr, g, s));
  else
    JAB_TRY(launch_attention(ws.qkv, ws.o, FMT_F16, batch, S, cfg->n_heads, cfg->head_dim,
                             padded ? ws.kv_len : nullptr, g, s));
  prof_mark(s, DIT_KERNEL_GEMM_O);
  JAB_TRY(launch_gemm_w8a16(GemmArgs{ws.o, FMT_F16, w->w_o, w->s_o, ws.x1, FMT_F32, x, FMT_BF16, M, d, d, 0, 0}, g, s));
  prof_mark(s, DIT_KERNEL_RMSNORM);
  if (w8a8)
    JAB_TRY(launch_rmsnorm_e4m3(ws.x1, FMT_F32, g2, h8, ws.sa, M, d, cfg->eps, s));
  else
    JAB_TRY(launch_rmsnorm(ws.x1, FMT_F32, g2, ws.h, FMT_F16, M, d, cfg->eps, s));
  prof_mark(s, DIT_KERNEL_GEMM_UP);
  if (w8a8)
    JAB_TRY(launch_gemm_w8a8(GemmArgs8{h8, ws.sa, w->w_up, w->s_up, ws.u, FMT_F16, M, F, d, 1, cfg->gelu_tanh}, g, s));
  else
    JAB_TRY(launch_gemm_w8a16(
        GemmArgs{ws.h, FMT_F16, w->w_up, w->s_up, ws.u, FMT_F16, nullptr, -1, M, F, d, 1, cfg->gelu_tanh}, g, s));
  prof_mark(s, DIT_KERNEL_GEMM_DOWN);
  JAB_TRY(launch_gemm_w8a16(
      GemmArgs{ws.u, FMT_F16, w->w_down, w->s_down, y, FMT_BF16, ws.x1, FMT_F32, M, d, F, 0, 0}, g, s));
  prof_mark(s, DIT_KERNEL_END);
#undef JAB_TRY
  return DIT_OK;
}

}  // namespace

extern "C" {

int dit_block_forward(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in, void* x_out,
                      int batch, int n_text, int grid_h, int grid_w, int t_img, const int32_t* pos, void* workspace,
                      size_t ws_bytes, void* stream) {
  return block_forward(cfg, w, x_in, x_out, batch, n_text, grid_h, grid_w, t_img, pos, nullptr, workspace, ws_bytes,
                       stream);
}

int dit_block_forward_w8a8(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in, void* x_out,
                           int batch, int n_text, int grid_h, int grid_w, int t_img, const int32_t* pos, void* workspace,
                           size_t ws_bytes, void* stream) {
  if (cfg != nullptr && cfg->d_model > 8192) return DIT_ERR_UNSUPPORTED;  // the e4m3 norm holds a row in registers
  return block_forward(cfg, w, x_in, x_out, batch, n_text, grid_h, grid_w, t_img, pos, nullptr, workspace, ws_bytes,
                       stream, true);
}

int dit_gemm_w8a8(const uint8_t* a8, const float* sa, const uint8_t* w8, const float* sw, void* y, int y_fmt, int M,
                  int N, int K, int act, int gelu_tanh, void* stream) {
  clear_stale_error();
  if (M < 0 || N <= 0 || K <= 0) return DIT_ERR_INVALID_ARG;
  if (N % 32 != 0 || K % 16 != 0) return DIT_ERR_UNSUPPORTED;
  if (y_fmt < FMT_BF16 || y_fmt > FMT_F32 || act < 0 || act > 1) return DIT_ERR_INVALID_ARG;
  if (M == 0) return DIT_OK;
  if (a8 == nullptr || sa == nullptr || w8 == nullptr || sw == nullptr || y == nullptr) return DIT_ERR_INVALID_ARG;
  if (!aligned16(a8) || !aligned16(w8) || !aligned16(y)) return DIT_ERR_INVALID_ARG;
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  return from_cuda(launch_gemm_w8a8(GemmArgs8{a8, sa, w8, sw, y, y_fmt, M, N, K, act, gelu_tanh}, g,
                                    as_stream(stream)));
}

int dit_rmsnorm_rows_e4m3(const void* x, int x_fmt, const void* g, uint8_t* y8, float* y_scale, int64_t rows,
                          int64_t cols, float eps, void* stream) {
  clear_stale_error();
  if (rows < 0 || cols <= 0 || cols % 8 != 0 || rows > (1ll << 31) - 1) return DIT_ERR_INVALID_ARG;
  if (cols > 8192) return DIT_ERR_UNSUPPORTED;
  if (x_fmt != FMT_BF16 && x_fmt != FMT_F32) return DIT_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || g == nullptr || y8 == nullptr || y_scale == nullptr)) return DIT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(g) || !aligned16(y8)) return DIT_ERR_INVALID_ARG;
  return from_cuda(launch_rmsnorm_e4m3(x, x_fmt, static_cast<const uint16_t*>(g), y8, y_scale, rows, cols, eps,
                                       as_stream(stream)));
}

int dit_block_forward_padded(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in, void* x_out,
                             int batch, int n_text, int grid_h, int grid_w, int t_img, const int32_t* text_lens,
                             void* workspace, size_t ws_bytes, void* stream) {
  if (text_lens == nullptr || !aligned16(text_lens)) return DIT_ERR_INVALID_ARG;
  return block_forward(cfg, w, x_in, x_out, batch, n_text, grid_h, grid_w, t_img, nullptr, text_lens, workspace,
                       ws_bytes, stream);
}

size_t dit_stack_workspace_bytes(const dit_block_config* cfg, int batch, int n_text, int grid_h, int grid_w) {
  const size_t blk = dit_block_workspace_bytes(cfg, batch, n_text, grid_h, grid_w);
  if (blk == 0) return 0;
  const size_t S = static_cast<size_t>(n_text) + static_cast<size_t>(grid_h) * grid_w;
  return blk + align256(static_cast<size_t>(batch) * S * cfg->d_model * 2);
}

int dit_stack_forward(const dit_block_config* cfg, const dit_block_weights* w, int n_blocks, const void* x_in,
                      void* x_out, int batch, int n_text, int grid_h, int grid_w, int t_img, const int32_t* pos,
                      void* workspace, size_t ws_bytes, void* stream) {
  int st = check_config(cfg);
  if (st != DIT_OK) return st;
  if (w == nullptr || n_blocks < 1 || x_in == nullptr || x_out == nullptr || x_in == x_out) return DIT_ERR_INVALID_ARG;
  if (!shape_ok(batch, n_text, grid_h, grid_w)) return DIT_ERR_INVALID_ARG;
  const size_t blk = dit_block_workspace_bytes(cfg, batch, n_text, grid_h, grid_w);
  const size_t need = dit_stack_workspace_bytes(cfg, batch, n_text, grid_h, grid_w);
  if (blk == 0 || need == 0) return DIT_ERR_UNSUPPORTED;
  if (workspace == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return DIT_ERR_WORKSPACE;
  void* buf = static_cast<uint8_t*>(workspace) + blk;  // [batch, S, d] bf16, ping-pong partner of x_out
  const void* in = x_in;
  for (int i = 0; i < n_blocks; ++i) {
    // block i writes x_out when (n_blocks - 1 - i) is even, so the last block lands in x_out
    void* out = ((n_blocks - 1 - i) & 1) == 0 ? x_out : buf;
    st = dit_block_forward(cfg, &w[i], in, out, batch, n_text, grid_h, grid_w, t_img, pos, workspace, blk, stream);
    if (st != DIT_OK) return st;
    in = out;
  }
  return DIT_OK;
}

size_t cond_proj_workspace_bytes(int n_tok, int n_layers, int hidden, int d_out) {
  if (n_tok <= 0 || n_layers <= 0 || hidden <= 0 || d_out <= 0) return 0;
  const int64_t K = static_cast<int64_t>(n_layers) * hidden;
  if (K > (1 << 30)) return 0;
  const int splits = gemm_pick_splits(n_tok, d_out, static_cast<int>(K));
  size_t bytes = align256(static_cast<size_t>(n_tok) * K * 2);
  if (splits > 1) bytes += align256(static_cast<size_t>(splits) * n_tok * d_out * 4);
  return bytes;
}

int cond_proj_forward(const void* feats, int n_tok, int n_layers, int hidden, const void* g_norm, float eps,
                      const uint8_t* w, const float* scale, int d_out, void* out, void* workspace, size_t ws_bytes,
                      void* stream) {
  clear_stale_error();
  if (n_tok <= 0 || n_layers <= 0 || hidden <= 0 || d_out <= 0) return DIT_ERR_INVALID_ARG;
  const int64_t K = static_cast<int64_t>(n_layers) * hidden;
  if (K % 256 != 0 || d_out % 256 != 0 || K > (1 << 30)) return DIT_ERR_UNSUPPORTED;
  if (feats == nullptr || g_norm == nullptr || w == nullptr || scale == nullptr || out == nullptr)
    return DIT_ERR_INVALID_ARG;
  if (!aligned16(feats) || !aligned16(g_norm) || !aligned16(w) || !aligned16(out)) return DIT_ERR_INVALID_ARG;
  const size_t need = cond_proj_workspace_bytes(n_tok, n_layers, hidden, d_out);
  if (workspace == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return DIT_ERR_WORKSPACE;
  KernelGuard g;
  if (current_guard(&g) != cudaSuccess) return DIT_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  uint16_t* normed = static_cast<uint16_t*>(workspace);  // f16 [n_tok, K]
  prof_mark(s, DIT_KERNEL_COND_RMSNORM);
  if (launch_rmsnorm(feats, FMT_BF16, static_cast<const uint16_t*>(g_norm), normed, FMT_F16, n_tok, K, eps, s) !=
      cudaSuccess)
    return DIT_ERR_CUDA;
  const int splits = gemm_pick_splits(n_tok, d_out, static_cast<int>(K));
  prof_mark(s, DIT_KERNEL_COND_GEMM);
  cudaError_t e;
  if (splits > 1) {
    float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                           align256(static_cast<size_t>(n_tok) * K * 2));
    GemmArgs ga{normed, FMT_F16, w, scale, part, FMT_F32, nullptr, -1, n_tok, d_out, static_cast<int>(K), 0, 0};
    ga.k_splits = splits;
    e = launch_gemm_w8a16(ga, g, s);
    if (e == cudaSuccess) {
      prof_mark(s, DIT_KERNEL_COND_REDUCE);
      e = launch_splitk_reduce(part, static_cast<uint16_t*>(out), static_cast<int64_t>(n_tok) * d_out, splits, s);
    }
  } else {
    e = launch_gemm_w8a16(
        GemmArgs{normed, FMT_F16, w, scale, out, FMT_BF16, nullptr, -1, n_tok, d_out, static_cast<int>(K), 0, 0}, g,
        s);
  }
  prof_mark(s, DIT_KERNEL_END);
  return from_cuda(e);
}


size_t dit_denoise_workspace_bytes(const dit_block_config* cfg, int batch, int n_text_c, int n_text_u, int grid_h,
                                   int grid_w) {
  const size_t sc = dit_stack_workspace_bytes(cfg, batch, n_text_c, grid_h, grid_w);
  const size_t su = dit_stack_workspace_bytes(cfg, batch, n_text_u, grid_h, grid_w);
  if (sc == 0 || su == 0 || grid_h * grid_w <= 0) return 0;
  const size_t n_img = static_cast<size_t>(grid_h) * grid_w;
  const size_t xc = align256(static_cast<size_t>(batch) * (n_text_c + n_img) * cfg->d_model * 2);
  const size_t xu = align256(static_cast<size_t>(batch) * (n_text_u + n_img) * cfg->d_model * 2);
  return 2 * xc + 2 * xu + (sc > su ? sc : su);
}

int dit_denoise_steps(const dit_block_config* cfg, const dit_block_weights* w_cond, const dit_block_weights* w_uncond,
                      int n_blocks, const void* text_cond, int n_text_c, const void* text_uncond, int n_text_u,
                      float* z, int batch, int grid_h, int grid_w, int n_steps, const float* guidance, const float* dt,
                      void* workspace, size_t ws_bytes, void* stream) {
  int st = check_config(cfg);
  if (st != DIT_OK) return st;
  if (w_cond == nullptr || w_uncond == nullptr || n_blocks < 1 || z == nullptr || n_steps < 0) return DIT_ERR_INVALID_ARG;
  if (n_steps > 0 && (guidance == nullptr || dt == nullptr)) return DIT_ERR_INVALID_ARG;
  if (grid_h <= 0 || grid_w <= 0 || n_text_c < 0 || n_text_u < 0) return DIT_ERR_INVALID_ARG;
  if ((n_text_c > 0 && text_cond == nullptr) || (n_text_u > 0 && text_uncond == nullptr)) return DIT_ERR_INVALID_ARG;
  if (!shape_ok(batch, n_text_c, grid_h, grid_w) || !shape_ok(batch, n_text_u, grid_h, grid_w))
    return DIT_ERR_INVALID_ARG;
  if (!aligned16(z) || !aligned16(text_cond) || !aligned16(text_uncond)) return DIT_ERR_INVALID_ARG;
  const size_t need = dit_denoise_workspace_bytes(cfg, batch, n_text_c, n_text_u, grid_h, grid_w);
  if (need == 0) return DIT_ERR_UNSUPPORTED;
  if (workspace == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return DIT_ERR_WORKSPACE;
  const int d = cfg->d_model, n_img = grid_h * grid_w;
  const size_t xc = align256(static_cast<size_t>(batch) * (n_text_c + n_img) * d * 2);
  const size_t xu = align256(static_cast<size_t>(batch) * (n_text_u + n_img) * d * 2);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint16_t* x_c = reinterpret_cast<uint16_t*>(base);
  uint16_t* out_c = reinterpret_cast<uint16_t*>(base + xc);
  uint16_t* x_u = reinterpret_cast<uint16_t*>(base + 2 * xc);
  uint16_t* out_u = reinterpret_cast<uint16_t*>(base + 2 * xc + xu);
  void* stack_ws = base + 2 * xc + 2 * xu;
  const size_t stack_bytes = ws_bytes - (2 * xc + 2 * xu);
  cudaStream_t s = as_stream(stream);
  for (int i = 0; i < n_steps; ++i) {
    if (launch_denoise_pack(z, static_cast<const uint16_t*>(text_cond), static_cast<const uint16_t*>(text_uncond), x_c,
                            x_u, batch, n_img, d, n_text_c, n_text_u, s) != cudaSuccess)
      return DIT_ERR_CUDA;
    st = dit_stack_forward(cfg, w_cond, n_blocks, x_c, out_c, batch, n_text_c, grid_h, grid_w, -1, nullptr, stack_ws,
                           stack_bytes, stream);
    if (st != DIT_OK) return st;
    st = dit_stack_forward(cfg, w_uncond, n_blocks, x_u, out_u, batch, n_text_u, grid_h, grid_w, -1, nullptr, stack_ws,
                           stack_bytes, stream);
    if (st != DIT_OK) return st;
    prof_mark(s, DIT_KERNEL_EULER_CFG);
    const cudaError_t e = launch_denoise_update(z, out_c, out_u, batch, n_img, d, n_text_c, n_text_u, guidance[i],
                                                dt[i], s);
    prof_mark(s, DIT_KERNEL_END);
    if (e != cudaSuccess) return DIT_ERR_CUDA;
  }
  return DIT_OK;
}

int dit_tokens_from_latent(const float* z, const void* text, void* x, int batch, int n_text, int n_img, int d_model,
                           void* stream) {
  clear_stale_error();
  if (batch <= 0 || n_text < 0 || n_img <= 0 || d_model <= 0 || d_model % 8 != 0) return DIT_ERR_INVALID_ARG;
  if (z == nullptr || x == nullptr || (n_text > 0 && text == nullptr)) return DIT_ERR_INVALID_ARG;
  if (!aligned16(z) || !aligned16(text) || !aligned16(x)) return DIT_ERR_INVALID_ARG;
  return from_cuda(launch_denoise_pack(z, static_cast<const uint16_t*>(text), nullptr, static_cast<uint16_t*>(x),
                                       nullptr, batch, n_img, d_model, n_text, 0, as_stream(stream)));
}

}  // extern "C"
