// Internal interfaces between the translation units of the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace jab {

// Launch with programmatic stream serialisation: the kernel may start while the previous
// kernel on the stream is finishing.  Every kernel launched this way executes
// griddepcontrol.wait (pdl_wait) before its first global-memory access, which returns once
// the previous kernel has completed and its writes are visible, and then
// griddepcontrol.launch_dependents, so the next kernel's CTAs can take the SMs its own tail
// leaves idle.  Outside such a chain the two instructions do nothing.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Passed by value to every kernel that waits: where to record errors and how long to wait.
struct KernelGuard {
  uint32_t* err;        // device error word of the current device
  uint64_t timeout_ns;  // wall-time limit of one bounded wait
};

// Device error codes (first one recorded wins).  0x1xx = a bounded wait timed out.
enum : uint32_t {
  ERR_NONE = 0,
  ERR_TIMEOUT_GEMM_PRODUCER = 0x101,
  ERR_TIMEOUT_GEMM_MMA = 0x102,
  ERR_TIMEOUT_GEMM_CONVERT = 0x103,
  ERR_TIMEOUT_GEMM_EPILOGUE = 0x104,
  ERR_TIMEOUT_GEMM_DRAIN = 0x105,
  ERR_TIMEOUT_GEMM_MMA_X = 0x106,
  ERR_TIMEOUT_GEMM_DRAIN_MMA = 0x107,
  ERR_TIMEOUT_ATTN_PRODUCER = 0x111,
  ERR_TIMEOUT_ATTN_MMA = 0x112,
  ERR_TIMEOUT_ATTN_SOFTMAX = 0x113,
  ERR_TIMEOUT_ATTN_DRAIN = 0x114,
  ERR_TIMEOUT_SELFTEST = 0x1F0,
};

// Guard for the current device (error word address + configured timeout).
cudaError_t current_guard(KernelGuard* g);

// TMA descriptor of a row-major tensor with up to 3 dims (dims[0] innermost, in elements).
bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base, const uint64_t* dims,
               const uint64_t* strides_bytes /* rank-1 entries */, const uint32_t* box, CUtensorMapSwizzle swz);

// ---- launchers (return cudaSuccess or the launch error) ----
cudaError_t launch_e4m3_to_bf16(const uint8_t* codes, uint16_t* out, int64_t n, cudaStream_t s);
// y = RMSNorm(x) * g; x in x_fmt (bf16 / f32), y in y_fmt (bf16 / f16), g bf16.
cudaError_t launch_rmsnorm(const void* x, int x_fmt, const uint16_t* g, void* y, int y_fmt, int64_t rows, int64_t cols,
                           float eps, cudaStream_t s);
cudaError_t launch_euler_cfg(float* x, const uint16_t* vc, const uint16_t* vu, int64_t n, float g, float dt,
                             cudaStream_t s);
// Denoising step: block inputs [text; bf16(latent)] of both branches, and the CFG + Euler update
// of the latent from the image rows of the two stacks' outputs.  d % 8 == 0.
cudaError_t launch_denoise_pack(const float* z, const uint16_t* text_c, const uint16_t* text_u, uint16_t* x_c,
                                uint16_t* x_u, int batch, int n_img, int d, int lc, int lu, cudaStream_t s);
cudaError_t launch_denoise_update(float* z, const uint16_t* out_c, const uint16_t* out_u, int batch, int n_img, int d,
                                  int lc, int lu, float guidance, float dt, cudaStream_t s);
cudaError_t launch_positions(int n_text, int grid_h, int grid_w, int t_img, int32_t* pos, cudaStream_t s);
// Per-head QK-RMSNorm + 3D M-RoPE in place on the fused qkv buffer; the rotary angles of each
// token are computed by the kernel from its position (text_lens / kv_len: padded batches).
cudaError_t launch_qknorm_mrope(void* qkv, int fmt, int batch, int seq, int n_heads, int head_dim, int n_text,
                                int grid_w, int n_img, int t_img, const int32_t* pos, const int32_t* text_lens,
                                int32_t* kv_len, const int32_t sections[3], float theta, const uint16_t* g_q,
                                const uint16_t* g_k, float eps, cudaStream_t s);

// Activation storage formats (the ABI's format codes).
enum Fmt : int { FMT_BF16 = 0, FMT_F16 = 1, FMT_F32 = 2 };

struct GemmArgs {
  const void* a;       // [M, K], a_fmt (bf16 or f16)
  int a_fmt;
  const uint8_t* w;    // e4m3 [N, K]
  const float* scale;  // [N]
  void* y;             // [M, N], y_fmt
  int y_fmt;
  const void* residual;  // [M, N], res_fmt, or null
  int res_fmt;
  int M, N, K;
  int act;        // 0 none, 1 GELU
  int gelu_tanh;
  int k_splits = 1;  // > 1: y is fp32 [k_splits, M, N] partial sums (scale applied; no act / residual)
};
cudaError_t launch_gemm_w8a16(const GemmArgs& args, const KernelGuard& g, cudaStream_t s);

// Y[M, N] = act( A8[M, K] (W8[N, K])^T * sa[m] * sw[n] ), e4m3 activations with a per-row scale and
// e4m3 weights with a per-row scale (tcgen05 kind::f8f6f4).  N % 32 == 0, K % 16 == 0.
struct GemmArgs8 {
  const uint8_t* a;  // e4m3 [M, K]
  const float* sa;   // [M]
  const uint8_t* w;  // e4m3 [N, K]
  const float* sw;   // [N]
  void* y;           // [M, N], y_fmt
  int y_fmt;
  int M, N, K;
  int act;  // 0 none, 1 GELU
  int gelu_tanh;
};
cudaError_t launch_gemm_w8a8(const GemmArgs8& args, const KernelGuard& g, cudaStream_t s);
// y8 = e4m3(RMSNorm(x) * g / s_row) with s_row = amax_row / 448 (1 for a zero row) written to ys;
// x in x_fmt (bf16 / f32); cols % 8 == 0 and cols <= 8192.
cudaError_t launch_rmsnorm_e4m3(const void* x, int x_fmt, const uint16_t* g, uint8_t* y8, float* ys, int64_t rows,
                                int64_t cols, float eps, cudaStream_t s);
// Split count that fills the SMs for an M x N x K problem (1 when the tile grid already does).
int gemm_pick_splits(int M, int N, int K);
// out (bf16, n elements) = sum of `splits` fp32 partials laid out [splits, n]; n % 8 == 0.
cudaError_t launch_splitk_reduce(const float* part, uint16_t* out, int64_t n, int splits, cudaStream_t s);

// qkv and out in fmt (bf16 or f16).
// A kernel whose only wait never completes (exercises the bounded-wait path).
cudaError_t launch_wait_selftest(const KernelGuard& g, cudaStream_t s);

// kv_len: optional device int32 [batch], the number of leading keys of each batch element that
// take part (clamped to [1, seq]); nullptr = all seq keys.
cudaError_t launch_attention(const void* qkv, void* out, int fmt, int batch, int seq, int n_heads, int head_dim,
                             const int32_t* kv_len, const KernelGuard& g, cudaStream_t s);

}  // namespace jab
