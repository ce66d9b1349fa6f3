// Pieces of the W8A8 variant's attention product with e4m3 q and k (q k^T on the tensor cores'
// 8-bit path; P V stays 16-bit).  Declared apart from internal.h: the 16-bit block path does not
// use them.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace jab {

// e4m3 outputs of the QK-norm kernel: q and k codes ([B * S, d] bytes each, 16-byte aligned) and
// their two static scales (scale[0]: q, scale[1]: k), fp32(fp32(sqrt(hd)) * max|g|) / 448.
struct QK8Out {
  uint8_t* q8;
  uint8_t* k8;
  float* scale;
};

// Per-head QK-RMSNorm + 3D M-RoPE of the fused qkv buffer as launch_qknorm_mrope computes them,
// written as e4m3 codes of value / scale into o8 instead of back into qkv (V is left as it is).
cudaError_t launch_qknorm_mrope_e4m3(const void* qkv, int fmt, int batch, int seq, int n_heads, int head_dim,
                                     int n_text, int grid_w, int n_img, int t_img, const int32_t* pos,
                                     const int32_t* text_lens, int32_t* kv_len, const int32_t sections[3], float theta,
                                     const uint16_t* g_q, const uint16_t* g_k, float eps, const QK8Out& o8,
                                     cudaStream_t s);

// Joint attention with e4m3 q8, k8 ([B, S, d] bytes) and the 16-bit V of the fused qkv buffer;
// S = scale[0] * scale[1] * (q8 k8^T), then softmax and P V as launch_attention does.
cudaError_t launch_attention_q8(const uint8_t* q8, const uint8_t* k8, const float* scale, const void* qkv, void* out,
                                int fmt, int batch, int seq, int n_heads, int head_dim, const int32_t* kv_len,
                                const KernelGuard& g, cudaStream_t s);

}  // namespace jab
