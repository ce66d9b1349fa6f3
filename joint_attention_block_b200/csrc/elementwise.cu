// HBM-bound kernels of the block: e4m3 -> bf16, row RMSNorm, the fused
// CFG + Euler update, the 3D M-RoPE position / angle tables and the standalone
// per-head QK-RMSNorm + M-RoPE.  All loads and stores are 16-byte vectors where
// the layout allows; math is fp32.
#include <cmath>

#include "common.cuh"
#include "qk8.h"

namespace jab {

// ------------------------------------------------------------------ e4m3 -> bf16

__global__ void e4m3_to_bf16_kernel(const uint8_t* __restrict__ codes, uint16_t* __restrict__ out, int64_t n) {
  const int64_t nvec = n / 16;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec; i += stride) {
    const uint4 v = reinterpret_cast<const uint4*>(codes)[i];
    uint4 o0, o1;
    e4m3x4_to_bf16x4(v.x, o0.x, o0.y);
    e4m3x4_to_bf16x4(v.y, o0.z, o0.w);
    e4m3x4_to_bf16x4(v.z, o1.x, o1.y);
    e4m3x4_to_bf16x4(v.w, o1.z, o1.w);
    reinterpret_cast<uint4*>(out)[2 * i] = o0;
    reinterpret_cast<uint4*>(out)[2 * i + 1] = o1;
  }
  // ragged tail, one code at a time
  const int64_t t = nvec * 16 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (t < n && blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x < 16) {
    uint32_t lo, hi;
    e4m3x4_to_bf16x4(codes[t], lo, hi);
    out[t] = static_cast<uint16_t>(lo & 0xFFFFu);
  }
}

cudaError_t launch_e4m3_to_bf16(const uint8_t* codes, uint16_t* out, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t nvec = n / 16;
  int blocks = static_cast<int>((nvec + 255) / 256);
  if (blocks < 1) blocks = 1;
  if (blocks > 148 * 16) blocks = 148 * 16;
  e4m3_to_bf16_kernel<<<blocks, 256, 0, s>>>(codes, out, n);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ RMSNorm rows

template <int kThreads>
__device__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = threadIdx.x < kThreads / 32 ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// One CTA per row.  kVec 8-element vectors per thread are kept in registers
// between the two passes when the row fits (cols <= kThreads*8*kVec); longer
// rows (the 53,248-wide conditioning features) are re-read from L2, four vectors
// per thread in flight in each pass.
// XF: input format (bf16 or fp32), YF: output format (bf16 or f16).
template <int kThreads, int kVec, int XF, int YF>
__global__ void __launch_bounds__(kThreads) rmsnorm_kernel(const void* x, const uint16_t* __restrict__ g, void* y,
                                                           int64_t cols, float eps) {
  pdl_wait_then_release();
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int64_t nv = cols / 8;
  const int64_t row8 = row * nv;
  float ss = 0.f;
  if constexpr (kVec > 0) {
    float v[kVec][8];
#pragma unroll
    for (int j = 0; j < kVec; ++j) {
      const int64_t i = threadIdx.x + static_cast<int64_t>(j) * kThreads;
      if (i < nv) {
        load8<XF>(x, row8 + i, v[j]);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[j][k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) ss = fmaf(v[j][k], v[j][k], ss);
    }
    const float rstd = rsqrtf(block_sum<kThreads>(ss, red) / static_cast<float>(cols) + eps);
#pragma unroll
    for (int j = 0; j < kVec; ++j) {
      const int64_t i = threadIdx.x + static_cast<int64_t>(j) * kThreads;
      if (i >= nv) break;
      float gv[8], o[8];
      load8<FMT_BF16>(g, i, gv);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = v[j][k] * rstd * gv[k];
      store8<YF>(y, row8 + i, o);
    }
  } else if constexpr (XF == FMT_F32) {
    for (int64_t i = threadIdx.x; i < nv; i += kThreads) {
      float v[8];
      load8<XF>(x, row8 + i, v);
#pragma unroll
      for (int k = 0; k < 8; ++k) ss = fmaf(v[k], v[k], ss);
    }
    const float rstd = rsqrtf(block_sum<kThreads>(ss, red) / static_cast<float>(cols) + eps);
    for (int64_t i = threadIdx.x; i < nv; i += kThreads) {
      float v[8], gv[8], o[8];
      load8<XF>(x, row8 + i, v);
      load8<FMT_BF16>(g, i, gv);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = v[k] * rstd * gv[k];
      store8<YF>(y, row8 + i, o);
    }
  } else {
    // 16-bit rows: U raw 16-byte vectors per thread in flight in each pass, unpacked as used
    constexpr int U = 4;
    const uint4* xr = reinterpret_cast<const uint4*>(x) + row8;
    const uint4* gr = reinterpret_cast<const uint4*>(g);
    for (int64_t i0 = threadIdx.x; i0 < nv; i0 += U * kThreads) {
      uint4 raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t i = i0 + static_cast<int64_t>(u) * kThreads;
        raw[u] = i < nv ? xr[i] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = unpack_lo<XF>(w[k]), b2 = unpack_hi<XF>(w[k]);
          ss = fmaf(a, a, fmaf(b2, b2, ss));
        }
      }
    }
    const float rstd = rsqrtf(block_sum<kThreads>(ss, red) / static_cast<float>(cols) + eps);
    for (int64_t i0 = threadIdx.x; i0 < nv; i0 += U * kThreads) {
      uint4 raw[U], graw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t i = i0 + static_cast<int64_t>(u) * kThreads;
        if (i < nv) {
          raw[u] = xr[i];
          graw[u] = gr[i];
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t i = i0 + static_cast<int64_t>(u) * kThreads;
        if (i < nv) {
          const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
          const uint32_t gw[4] = {graw[u].x, graw[u].y, graw[u].z, graw[u].w};
          float o[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            o[2 * k] = unpack_lo<XF>(w[k]) * rstd * unpack_lo<FMT_BF16>(gw[k]);
            o[2 * k + 1] = unpack_hi<XF>(w[k]) * rstd * unpack_hi<FMT_BF16>(gw[k]);
          }
          store8<YF>(y, row8 + i, o);
        }
      }
    }
  }
}

template <int XF, int YF>
static void rmsnorm_dispatch(const void* x, const uint16_t* g, void* y, int64_t rows, int64_t cols, float eps,
                             cudaStream_t s) {
  const unsigned r = static_cast<unsigned>(rows);
  if (cols <= 256 * 8 * 1) {
    launch_pdl(rmsnorm_kernel<256, 1, XF, YF>, dim3(r), dim3(256), 0, s, x, g, y, cols, eps);
  } else if (cols <= 256 * 8 * 2) {
    launch_pdl(rmsnorm_kernel<256, 2, XF, YF>, dim3(r), dim3(256), 0, s, x, g, y, cols, eps);
  } else if (cols <= 256 * 8 * 4) {
    launch_pdl(rmsnorm_kernel<256, 4, XF, YF>, dim3(r), dim3(256), 0, s, x, g, y, cols, eps);
  } else {
    launch_pdl(rmsnorm_kernel<512, 0, XF, YF>, dim3(r), dim3(512), 0, s, x, g, y, cols, eps);
  }
}

cudaError_t launch_rmsnorm(const void* x, int x_fmt, const uint16_t* g, void* y, int y_fmt, int64_t rows, int64_t cols,
                           float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (x_fmt == FMT_BF16 && y_fmt == FMT_BF16) rmsnorm_dispatch<FMT_BF16, FMT_BF16>(x, g, y, rows, cols, eps, s);
  else if (x_fmt == FMT_BF16 && y_fmt == FMT_F16) rmsnorm_dispatch<FMT_BF16, FMT_F16>(x, g, y, rows, cols, eps, s);
  else if (x_fmt == FMT_F32 && y_fmt == FMT_F16) rmsnorm_dispatch<FMT_F32, FMT_F16>(x, g, y, rows, cols, eps, s);
  else if (x_fmt == FMT_F32 && y_fmt == FMT_BF16) rmsnorm_dispatch<FMT_F32, FMT_BF16>(x, g, y, rows, cols, eps, s);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ RMSNorm to per-token e4m3

template <int kThreads>
__device__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = threadIdx.x < kThreads / 32 ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// Two fp32 -> packed e4m3x2 (round to nearest even, saturating at +-448), lo in the low byte.
__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// One CTA per row, the row held in registers: o = x / sqrt(mean(x^2) + eps) * g in fp32, then
// the row's scale s = amax(|o|) / 448 and codes e4m3(o / s) (IEEE division, then round to nearest
// even).  The scale goes to ys[row].
template <int kThreads, int kVec, int XF>
__global__ void __launch_bounds__(kThreads) rmsnorm_e4m3_kernel(const void* x, const uint16_t* __restrict__ g,
                                                                uint8_t* __restrict__ y8, float* __restrict__ ys,
                                                                int64_t cols, float eps) {
  pdl_wait_then_release();
  __shared__ float red[32];
  __shared__ float red2[32];
  const int64_t row = blockIdx.x;
  const int64_t nv = cols / 8;
  float v[kVec][8];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int64_t i = threadIdx.x + static_cast<int64_t>(j) * kThreads;
    if (i < nv) {
      load8<XF>(x, row * nv + i, v[j]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[j][k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) ss = fmaf(v[j][k], v[j][k], ss);
  }
  const float rstd = rsqrtf(block_sum<kThreads>(ss, red) / static_cast<float>(cols) + eps);
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int64_t i = threadIdx.x + static_cast<int64_t>(j) * kThreads;
    float gv[8];
    if (i < nv) {
      load8<FMT_BF16>(g, i, gv);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) gv[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[j][k] = v[j][k] * rstd * gv[k];
      amax = fmaxf(amax, fabsf(v[j][k]));
    }
  }
  amax = block_max<kThreads>(amax, red2);
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  if (threadIdx.x == 0) ys[row] = scale;
#pragma unroll
  for (int j = 0; j < kVec; ++j) {
    const int64_t i = threadIdx.x + static_cast<int64_t>(j) * kThreads;
    if (i >= nv) break;
    uint2 o;
    o.x = static_cast<uint32_t>(pack_e4m3x2(v[j][0] / scale, v[j][1] / scale)) |
          (static_cast<uint32_t>(pack_e4m3x2(v[j][2] / scale, v[j][3] / scale)) << 16);
    o.y = static_cast<uint32_t>(pack_e4m3x2(v[j][4] / scale, v[j][5] / scale)) |
          (static_cast<uint32_t>(pack_e4m3x2(v[j][6] / scale, v[j][7] / scale)) << 16);
    reinterpret_cast<uint2*>(y8)[row * nv + i] = o;
  }
}

template <int XF>
static void rmsnorm_e4m3_dispatch(const void* x, const uint16_t* g, uint8_t* y8, float* ys, int64_t rows,
                                  int64_t cols, float eps, cudaStream_t s) {
  const unsigned r = static_cast<unsigned>(rows);
  if (cols <= 256 * 8 * 1)
    launch_pdl(rmsnorm_e4m3_kernel<256, 1, XF>, dim3(r), dim3(256), 0, s, x, g, y8, ys, cols, eps);
  else if (cols <= 256 * 8 * 2)
    launch_pdl(rmsnorm_e4m3_kernel<256, 2, XF>, dim3(r), dim3(256), 0, s, x, g, y8, ys, cols, eps);
  else
    launch_pdl(rmsnorm_e4m3_kernel<256, 4, XF>, dim3(r), dim3(256), 0, s, x, g, y8, ys, cols, eps);
}

cudaError_t launch_rmsnorm_e4m3(const void* x, int x_fmt, const uint16_t* g, uint8_t* y8, float* ys, int64_t rows,
                                int64_t cols, float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (cols % 8 != 0 || cols > 256 * 8 * 4) return cudaErrorInvalidValue;
  if (x_fmt == FMT_BF16) rmsnorm_e4m3_dispatch<FMT_BF16>(x, g, y8, ys, rows, cols, eps, s);
  else if (x_fmt == FMT_F32) rmsnorm_e4m3_dispatch<FMT_F32>(x, g, y8, ys, rows, cols, eps, s);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ CFG + Euler

// x <- x + dt * (v_u + g * (v_c - v_u)); 8 elements per thread per iteration.
__global__ void euler_cfg_kernel(float* __restrict__ x, const uint16_t* __restrict__ vc,
                                 const uint16_t* __restrict__ vu, int64_t n, float guidance, float dt) {
  pdl_wait_then_release();
  const int64_t nvec = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec; i += stride) {
    float4 x0 = reinterpret_cast<const float4*>(x)[2 * i];
    float4 x1 = reinterpret_cast<const float4*>(x)[2 * i + 1];
    const uint4 c = reinterpret_cast<const uint4*>(vc)[i];
    const uint4 u = reinterpret_cast<const uint4*>(vu)[i];
    float* xs0 = reinterpret_cast<float*>(&x0);
    float* xs1 = reinterpret_cast<float*>(&x1);
    const uint32_t* cs = reinterpret_cast<const uint32_t*>(&c);
    const uint32_t* us = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float* xk = k < 2 ? xs0 + 2 * k : xs1 + 2 * (k - 2);
      const float c0 = bf16_lo(cs[k]), c1 = bf16_hi(cs[k]);
      const float u0 = bf16_lo(us[k]), u1 = bf16_hi(us[k]);
      xk[0] = fmaf(dt, fmaf(guidance, c0 - u0, u0), xk[0]);
      xk[1] = fmaf(dt, fmaf(guidance, c1 - u1, u1), xk[1]);
    }
    reinterpret_cast<float4*>(x)[2 * i] = x0;
    reinterpret_cast<float4*>(x)[2 * i + 1] = x1;
  }
  const int64_t t = nvec * 8 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (t < n && blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x < 8) {
    const float c0 = __uint_as_float(static_cast<uint32_t>(vc[t]) << 16);
    const float u0 = __uint_as_float(static_cast<uint32_t>(vu[t]) << 16);
    x[t] = fmaf(dt, fmaf(guidance, c0 - u0, u0), x[t]);
  }
}

cudaError_t launch_euler_cfg(float* x, const uint16_t* vc, const uint16_t* vu, int64_t n, float g, float dt,
                             cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t nvec = n / 8;
  int64_t blocks = (nvec + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 148 * 8) blocks = 148 * 8;
  launch_pdl(euler_cfg_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, x, vc, vu, n, g, dt);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ denoising step: latent <-> tokens

// Block inputs of one denoising step: for every batch element, x_c = [text_c; bf16(z)] and
// x_u = [text_u; bf16(z)] (the latent's rows are the image tokens).  One thread per 8 values
// of one row of x_c (the uncond rows are written by the same thread when they exist); x_u may
// be null (one branch only).
__global__ void denoise_pack_kernel(const float* __restrict__ z, const uint16_t* __restrict__ text_c,
                                    const uint16_t* __restrict__ text_u, uint16_t* __restrict__ x_c,
                                    uint16_t* __restrict__ x_u, int batch, int n_img, int d, int lc, int lu) {
  pdl_wait_then_release();
  const int v8 = d / 8;
  const int rows = max(lc, lu) + n_img;
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= static_cast<int64_t>(batch) * rows * v8) return;
  const int c = static_cast<int>(idx % v8);
  const int64_t br = idx / v8;
  const int b = static_cast<int>(br / rows);
  const int r = static_cast<int>(br % rows);  // r < n_img: image row r; otherwise text row r - n_img
  if (r < n_img) {
    float v[8];
    load8<FMT_F32>(z, (static_cast<int64_t>(b) * n_img + r) * v8 + c, v);
    store8<FMT_BF16>(x_c, (static_cast<int64_t>(b) * (lc + n_img) + lc + r) * v8 + c, v);
    if (x_u != nullptr) store8<FMT_BF16>(x_u, (static_cast<int64_t>(b) * (lu + n_img) + lu + r) * v8 + c, v);
  } else {
    const int t = r - n_img;
    const uint4* src;
    if (t < lc) {
      src = reinterpret_cast<const uint4*>(text_c) + (static_cast<int64_t>(b) * lc + t) * v8 + c;
      reinterpret_cast<uint4*>(x_c)[(static_cast<int64_t>(b) * (lc + n_img) + t) * v8 + c] = *src;
    }
    if (t < lu && x_u != nullptr) {
      src = reinterpret_cast<const uint4*>(text_u) + (static_cast<int64_t>(b) * lu + t) * v8 + c;
      reinterpret_cast<uint4*>(x_u)[(static_cast<int64_t>(b) * (lu + n_img) + t) * v8 + c] = *src;
    }
  }
}

cudaError_t launch_denoise_pack(const float* z, const uint16_t* text_c, const uint16_t* text_u, uint16_t* x_c,
                                uint16_t* x_u, int batch, int n_img, int d, int lc, int lu, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(batch) * (max(lc, lu) + n_img) * (d / 8);
  if (n <= 0) return cudaSuccess;
  launch_pdl(denoise_pack_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, s, z, text_c, text_u,
             x_c, x_u, batch, n_img, d, lc, lu);
  return cudaGetLastError();
}

// z[b, i] += dt * (v_u + g (v_c - v_u)) with v_c = out_c[b, lc + i] and v_u = out_u[b, lu + i]
// (the image rows of the two stacks' outputs), the fp32 arithmetic of euler_cfg_kernel.
__global__ void denoise_update_kernel(float* __restrict__ z, const uint16_t* __restrict__ out_c,
                                      const uint16_t* __restrict__ out_u, int batch, int n_img, int d, int lc, int lu,
                                      float guidance, float dt) {
  pdl_wait_then_release();
  const int v8 = d / 8;
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= static_cast<int64_t>(batch) * n_img * v8) return;
  const int c = static_cast<int>(idx % v8);
  const int64_t bi = idx / v8;
  const int b = static_cast<int>(bi / n_img);
  const int i = static_cast<int>(bi % n_img);
  float x[8], vc[8], vu[8];
  load8<FMT_F32>(z, idx, x);
  load8<FMT_BF16>(out_c, (static_cast<int64_t>(b) * (lc + n_img) + lc + i) * v8 + c, vc);
  load8<FMT_BF16>(out_u, (static_cast<int64_t>(b) * (lu + n_img) + lu + i) * v8 + c, vu);
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = fmaf(dt, fmaf(guidance, vc[k] - vu[k], vu[k]), x[k]);
  store8<FMT_F32>(z, idx, x);
}

cudaError_t launch_denoise_update(float* z, const uint16_t* out_c, const uint16_t* out_u, int batch, int n_img, int d,
                                  int lc, int lu, float guidance, float dt, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(batch) * n_img * (d / 8);
  if (n <= 0) return cudaSuccess;
  launch_pdl(denoise_update_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, s, z, out_c, out_u,
             batch, n_img, d, lc, lu, guidance, dt);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ positions and angle tables

// Text token j -> (j, j, j); image cell (r, c) in raster order -> (t_img, r, c).
// Positions and inverse frequencies of the rotary embedding, passed by value to the QK-norm kernel.
struct RopeArgs {
  int n_text, grid_w, n_img, t_img;  // t_img < 0: n_text (or L_b in a padded batch)
  const int32_t* pos;                // [S, 3] or NULL (ignored when text_lens is given)
  const int32_t* text_lens;          // [batch] or NULL
  int32_t* kv_len;                   // [batch], written when text_lens is given
  int sec_t, sec_h;                  // rotary pairs on the t and h axes (w takes the rest)
  float inv_freq[64];                // fp32(theta^(-2i/hd)), i < hd/2
};

__device__ __forceinline__ void token_position(int s, int n_text, int grid_w, int t_img, const int32_t* pos, int& pt,
                                               int& ph, int& pw) {
  if (pos != nullptr) {
    pt = pos[3 * s];
    ph = pos[3 * s + 1];
    pw = pos[3 * s + 2];
  } else if (s < n_text) {
    pt = ph = pw = s;
  } else {
    const int i = s - n_text;
    pt = t_img;
    ph = i / grid_w;
    pw = i - ph * grid_w;
  }
}

__global__ void positions_kernel(int n_text, int grid_h, int grid_w, int t_img, int32_t* pos) {
  const int S = n_text + grid_h * grid_w;
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= S) return;
  int pt, ph, pw;
  token_position(s, n_text, grid_w, t_img, nullptr, pt, ph, pw);
  pos[3 * s] = pt;
  pos[3 * s + 1] = ph;
  pos[3 * s + 2] = pw;
}

cudaError_t launch_positions(int n_text, int grid_h, int grid_w, int t_img, int32_t* pos, cudaStream_t s) {
  const int S = n_text + grid_h * grid_w;
  if (S <= 0) return cudaSuccess;
  positions_kernel<<<(S + 255) / 256, 256, 0, s>>>(n_text, grid_h, grid_w, t_img, pos);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ QK-RMSNorm + M-RoPE

// One CTA per (batch element b, token s).  The token's rotary angles come first: for pair i
// (i < hd/2) the position on axis(i) (t for the first sec_t pairs, then h for sec_h, then w)
// times inv_freq_i = fp32(theta^(-2i/hd)) (exact in fp64), reduced modulo 2 pi in fp64, and its
// cosine and sine in fp32 (within a few fp32 ulps of the fp64 values), into shared memory.  Positions: text j at (j, j, j), image cell
// (r, c) at (t_img, r, c), or the caller's pos[s]; in a padded batch (text_lens given) element
// b has L_b = clamp(text_lens[b], 0, n_text) text rows, then its image rows at (t_b, r, c),
// t_b = L_b (or t_img when t_img >= 0), then padding at (0, 0, 0), and the CTA of (b, 0) also
// writes the element's key count L_b + n_img to kv_len[b].
// Then one thread per (head, 8 rotary pairs): it holds elements [8c, 8c+8) and
// [half+8c, half+8c+8) of the head in both q and k as 16-byte vectors (loaded before the
// angles are computed), so the hd/16 threads of one head are consecutive lanes and reduce the
// two sums of squares with xor-shuffles.  The CTA is a whole number of warps; lanes past the
// last head shadow it so that the shuffles stay full.  F: storage format of the qkv buffer.
// Q8 (the W8A8 variant): q and k are not written back; their e4m3 codes go to o8.q8 / o8.k8
// ([B * S, d] bytes), each divided by one static scale, fp32(fp32(sqrt(hd)) * max|g|) / 448 (the
// norm of a normalised head vector is at most sqrt(hd) * max|g| and the rotations keep it, so no
// code saturates), which the CTA of token 0 also stores in o8.scale[0] (q) and [1] (k).
template <int F, bool Q8>
__global__ void __launch_bounds__(512, 2)  // <= 64 registers: four 256-thread CTAs per SM
    qknorm_mrope_kernel(uint16_t* __restrict__ qkv, int seq, int n_heads, int head_dim, RopeArgs ra,
                                    const uint16_t* __restrict__ g_q, const uint16_t* __restrict__ g_k, float eps,
                                    QK8Out o8) {
  __shared__ float s_cos[64], s_sin[64];
  __shared__ float s_gmax[2];  // Q8: max |g_q|, max |g_k|
  pdl_wait_then_release();
  const int half = head_dim / 2;
  const int lg = head_dim == 128 ? 3 : 2;  // log2 of the threads per head: 8 (hd 128) or 4 (hd 64)
  const int group = 1 << lg;
  const int per_token = n_heads << lg;
  const bool live = static_cast<int>(threadIdx.x) < per_token;
  const int t = live ? static_cast<int>(threadIdx.x) : per_token - 1;
  const int c = t & (group - 1);
  const int h = t >> lg;
  const int64_t bs = blockIdx.x;  // b * seq + s
  const int b = static_cast<int>(bs / seq);
  const int s = static_cast<int>(bs - static_cast<int64_t>(b) * seq);
  const int d = n_heads * head_dim;
  uint16_t* vq = qkv + bs * (3 * static_cast<int64_t>(d)) + h * head_dim;
  uint16_t* vk = vq + d;
  // q and k halves stay packed (8 16-bit values per 16-byte vector) until they are used
  const uint4 rqa = *reinterpret_cast<const uint4*>(vq + 8 * c);
  const uint4 rqb = *reinterpret_cast<const uint4*>(vq + half + 8 * c);
  const uint4 rka = *reinterpret_cast<const uint4*>(vk + 8 * c);
  const uint4 rkb = *reinterpret_cast<const uint4*>(vk + half + 8 * c);
  {
    int pt = 0, ph = 0, pw = 0;
    if (ra.text_lens != nullptr) {
      const int L = min(max(ra.text_lens[b], 0), ra.n_text);
      if (s == 0 && threadIdx.x == 0) ra.kv_len[b] = L + ra.n_img;
      if (s < L) {
        pt = ph = pw = s;
      } else if (s < L + ra.n_img) {
        const int k = s - L;
        pt = ra.t_img < 0 ? L : ra.t_img;
        ph = k / ra.grid_w;
        pw = k - ph * ra.grid_w;
      }
    } else {
      token_position(s, ra.n_text, ra.grid_w, ra.t_img < 0 ? ra.n_text : ra.t_img, ra.pos, pt, ph, pw);
    }
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      const int p = i < ra.sec_t ? pt : (i < ra.sec_t + ra.sec_h ? ph : pw);
      // the angle p * inv_freq_i is exact in fp64; it is reduced by the nearest multiple of 2 pi
      // in fp64 (error ~1e-13 for the angles of any image), rounded once to fp32 in [-pi, pi],
      // and its sine and cosine taken in fp32
      const double x = static_cast<double>(p) * static_cast<double>(ra.inv_freq[i]);
      const double k = rint(x * 0.15915494309189535);
      const float r = static_cast<float>(fma(-k, 6.283185307179586, x));
      float sn, cs;
      sincosf(r, &sn, &cs);
      s_cos[i] = cs;
      s_sin[i] = sn;
    }
  }
  if constexpr (Q8) {
    if (threadIdx.x < 32) {  // max |g| of both gains, hd <= 128 values each: four per lane
      float mq = 0.f, mk = 0.f;
      for (int i = static_cast<int>(threadIdx.x); i < head_dim; i += 32) {
        mq = fmaxf(mq, fabsf(__uint_as_float(static_cast<uint32_t>(g_q[i]) << 16)));
        mk = fmaxf(mk, fabsf(__uint_as_float(static_cast<uint32_t>(g_k[i]) << 16)));
      }
      for (int o = 16; o > 0; o >>= 1) {
        mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
        mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
      }
      if (threadIdx.x == 0) {
        s_gmax[0] = mq;
        s_gmax[1] = mk;
      }
    }
  }
  auto sumsq = [](const uint4& a, const uint4& b2) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b2.x, b2.y, b2.z, b2.w};
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float lo = unpack_lo<F>(w[k]), hi = unpack_hi<F>(w[k]);
      acc = fmaf(lo, lo, fmaf(hi, hi, acc));
    }
    return acc;
  };
  float sq = sumsq(rqa, rqb), sk = sumsq(rka, rkb);
  for (int o = group / 2; o > 0; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    sk += __shfl_xor_sync(0xffffffffu, sk, o);
  }
  const float rq = rsqrtf(sq / static_cast<float>(head_dim) + eps);
  const float rk = rsqrtf(sk / static_cast<float>(head_dim) + eps);
  __syncthreads();  // the token's angles are in shared memory
  // rotate pairs (i, i + hd/2): x1 = a * r * g_a, x2 = b * r * g_b; (x1 cos - x2 sin, x2 cos + x1 sin)
  auto rotate = [&](const uint4& a, const uint4& b2, float rr, const uint16_t* g, uint16_t* dst) {
    const uint4 ga4 = *reinterpret_cast<const uint4*>(g + 8 * c);
    const uint4 gb4 = *reinterpret_cast<const uint4*>(g + half + 8 * c);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b2.x, b2.y, b2.z, b2.w};
    const uint32_t wga[4] = {ga4.x, ga4.y, ga4.z, ga4.w}, wgb[4] = {gb4.x, gb4.y, gb4.z, gb4.w};
    uint4 oa, ob;
    uint32_t* poa = reinterpret_cast<uint32_t*>(&oa);
    uint32_t* pob = reinterpret_cast<uint32_t*>(&ob);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float ra2[2], rb2[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 8 * c + 2 * k + e;
        const float av = e ? unpack_hi<F>(wa[k]) : unpack_lo<F>(wa[k]);
        const float bv = e ? unpack_hi<F>(wb[k]) : unpack_lo<F>(wb[k]);
        const float gav = e ? unpack_hi<FMT_BF16>(wga[k]) : unpack_lo<FMT_BF16>(wga[k]);
        const float gbv = e ? unpack_hi<FMT_BF16>(wgb[k]) : unpack_lo<FMT_BF16>(wgb[k]);
        const float x1 = av * rr * gav;
        const float x2 = bv * rr * gbv;
        const float cs = s_cos[i], sn = s_sin[i];
        ra2[e] = x1 * cs - x2 * sn;
        rb2[e] = x2 * cs + x1 * sn;
      }
      poa[k] = pack2<F>(ra2[0], ra2[1]);
      pob[k] = pack2<F>(rb2[0], rb2[1]);
    }
    *reinterpret_cast<uint4*>(dst + 8 * c) = oa;
    *reinterpret_cast<uint4*>(dst + half + 8 * c) = ob;
  };
  if constexpr (!Q8) {
    if (live) {
      rotate(rqa, rqb, rq, g_q, vq);
      rotate(rka, rkb, rk, g_k, vk);
    }
  } else {
    const float root = __fsqrt_rn(static_cast<float>(head_dim));
    const float sc_q = __fdiv_rn(__fmul_rn(root, s_gmax[0]), 448.f);  // after the __syncthreads above
    const float sc_k = __fdiv_rn(__fmul_rn(root, s_gmax[1]), 448.f);
    if (bs == 0 && threadIdx.x == 0) {
      o8.scale[0] = sc_q;
      o8.scale[1] = sc_k;
    }
    // the same rotation as above, then e4m3 codes of value * fp32(1 / scale) (8 bytes per half)
    auto rotate8 = [&](const uint4& a, const uint4& b2, float rr, const uint16_t* g, float inv, uint8_t* dst) {
      const uint4 ga4 = *reinterpret_cast<const uint4*>(g + 8 * c);
      const uint4 gb4 = *reinterpret_cast<const uint4*>(g + half + 8 * c);
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b2.x, b2.y, b2.z, b2.w};
      const uint32_t wga[4] = {ga4.x, ga4.y, ga4.z, ga4.w}, wgb[4] = {gb4.x, gb4.y, gb4.z, gb4.w};
      uint16_t ca[4], cb[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float ra2[2], rb2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 8 * c + 2 * k + e;
          const float av = e ? unpack_hi<F>(wa[k]) : unpack_lo<F>(wa[k]);
          const float bv = e ? unpack_hi<F>(wb[k]) : unpack_lo<F>(wb[k]);
          const float gav = e ? unpack_hi<FMT_BF16>(wga[k]) : unpack_lo<FMT_BF16>(wga[k]);
          const float gbv = e ? unpack_hi<FMT_BF16>(wgb[k]) : unpack_lo<FMT_BF16>(wgb[k]);
          const float x1 = av * rr * gav;
          const float x2 = bv * rr * gbv;
          const float cs = s_cos[i], sn = s_sin[i];
          ra2[e] = (x1 * cs - x2 * sn) * inv;
          rb2[e] = (x2 * cs + x1 * sn) * inv;
        }
        ca[k] = pack_e4m3x2(ra2[0], ra2[1]);
        cb[k] = pack_e4m3x2(rb2[0], rb2[1]);
      }
      *reinterpret_cast<uint2*>(dst + 8 * c) =
          make_uint2(ca[0] | (static_cast<uint32_t>(ca[1]) << 16), ca[2] | (static_cast<uint32_t>(ca[3]) << 16));
      *reinterpret_cast<uint2*>(dst + half + 8 * c) =
          make_uint2(cb[0] | (static_cast<uint32_t>(cb[1]) << 16), cb[2] | (static_cast<uint32_t>(cb[3]) << 16));
    };
    if (live) {
      const int64_t row = bs * static_cast<int64_t>(d) + h * head_dim;
      rotate8(rqa, rqb, rq, g_q, __fdiv_rn(1.f, sc_q), o8.q8 + row);
      rotate8(rka, rkb, rk, g_k, __fdiv_rn(1.f, sc_k), o8.k8 + row);
    }
  }
}

namespace {

cudaError_t qknorm_mrope_impl(void* qkv, int fmt, int batch, int seq, int n_heads, int head_dim, int n_text,
                              int grid_w, int n_img, int t_img, const int32_t* pos, const int32_t* text_lens,
                              int32_t* kv_len, const int32_t sections[3], float theta, const uint16_t* g_q,
                              const uint16_t* g_k, float eps, cudaStream_t s, const QK8Out* o8) {
  const int64_t tokens = static_cast<int64_t>(batch) * seq;
  if (tokens <= 0 || n_heads <= 0) return cudaSuccess;
  if (head_dim != 64 && head_dim != 128) return cudaErrorInvalidValue;
  if ((text_lens != nullptr) != (kv_len != nullptr)) return cudaErrorInvalidValue;
  const int per_token = n_heads * (head_dim / 16);
  if (per_token > 512) return cudaErrorInvalidValue;  // the kernel's launch bound
  RopeArgs ra;
  ra.n_text = n_text;
  ra.grid_w = grid_w > 0 ? grid_w : 1;
  ra.n_img = n_img;
  ra.t_img = t_img;
  ra.pos = pos;
  ra.text_lens = text_lens;
  ra.kv_len = kv_len;
  ra.sec_t = sections[0];
  ra.sec_h = sections[1];
  for (int i = 0; i < head_dim / 2; ++i)
    ra.inv_freq[i] = static_cast<float>(std::pow(static_cast<double>(theta), -2.0 * i / head_dim));
  const unsigned threads = static_cast<unsigned>((per_token + 31) / 32 * 32);
  const unsigned blocks = static_cast<unsigned>(tokens);
  uint16_t* q = static_cast<uint16_t*>(qkv);
  if (o8 != nullptr) {
    if (o8->q8 == nullptr || o8->k8 == nullptr || o8->scale == nullptr) return cudaErrorInvalidValue;
    if (((reinterpret_cast<uintptr_t>(o8->q8) | reinterpret_cast<uintptr_t>(o8->k8)) & 15u) != 0)
      return cudaErrorInvalidValue;
    if (fmt == FMT_F16)
      launch_pdl(qknorm_mrope_kernel<FMT_F16, true>, dim3(blocks), dim3(threads), 0, s, q, seq, n_heads, head_dim, ra,
                 g_q, g_k, eps, *o8);
    else if (fmt == FMT_BF16)
      launch_pdl(qknorm_mrope_kernel<FMT_BF16, true>, dim3(blocks), dim3(threads), 0, s, q, seq, n_heads, head_dim, ra,
                 g_q, g_k, eps, *o8);
    else
      return cudaErrorInvalidValue;
    return cudaGetLastError();
  }
  const QK8Out none{nullptr, nullptr, nullptr};
  if (fmt == FMT_F16)
    launch_pdl(qknorm_mrope_kernel<FMT_F16, false>, dim3(blocks), dim3(threads), 0, s, q, seq, n_heads, head_dim, ra,
               g_q, g_k, eps, none);
  else if (fmt == FMT_BF16)
    launch_pdl(qknorm_mrope_kernel<FMT_BF16, false>, dim3(blocks), dim3(threads), 0, s, q, seq, n_heads, head_dim, ra,
               g_q, g_k, eps, none);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qknorm_mrope(void* qkv, int fmt, int batch, int seq, int n_heads, int head_dim, int n_text,
                                int grid_w, int n_img, int t_img, const int32_t* pos, const int32_t* text_lens,
                                int32_t* kv_len, const int32_t sections[3], float theta, const uint16_t* g_q,
                                const uint16_t* g_k, float eps, cudaStream_t s) {
  return qknorm_mrope_impl(qkv, fmt, batch, seq, n_heads, head_dim, n_text, grid_w, n_img, t_img, pos, text_lens,
                           kv_len, sections, theta, g_q, g_k, eps, s, nullptr);
}

cudaError_t launch_qknorm_mrope_e4m3(const void* qkv, int fmt, int batch, int seq, int n_heads, int head_dim,
                                     int n_text, int grid_w, int n_img, int t_img, const int32_t* pos,
                                     const int32_t* text_lens, int32_t* kv_len, const int32_t sections[3], float theta,
                                     const uint16_t* g_q, const uint16_t* g_k, float eps, const QK8Out& o8,
                                     cudaStream_t s) {
  return qknorm_mrope_impl(const_cast<void*>(qkv), fmt, batch, seq, n_heads, head_dim, n_text, grid_w, n_img, t_img,
                           pos, text_lens, kv_len, sections, theta, g_q, g_k, eps, s, &o8);
}

// ------------------------------------------------------------------ bounded-wait self test

// One thread waits on an mbarrier that nothing arrives on; the bounded wait must give
// up after the guard's limit and record ERR_TIMEOUT_SELFTEST, leaving the context usable.
__global__ void wait_selftest_kernel(const KernelGuard guard) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0u;
  fence_barrier_init();
  mbar_wait(&bar, 0u, guard, &abort_flag, ERR_TIMEOUT_SELFTEST);
}

cudaError_t launch_wait_selftest(const KernelGuard& g, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(g);
  return cudaGetLastError();
}

}  // namespace jab
