// The LLaMA block around the SERQ linears, for the time-to-first-token of a
// 2K-token prefill (the measurement the reading notes report under
// "GPU 性能分析"): rotary position embedding, causal grouped-query attention
// in bf16, and the residual add. The pages do not restate these layers; they
// follow the standard LLaMA definitions:
//   RoPE (rotate-half): for pair i < d/2 of a head at position p,
//       angle = p * base^(-2i/d), (x_i, x_{i+d/2}) <- (x_i c - x_{i+d/2} s, x_{i+d/2} c + x_i s)
//   attention: O_h = softmax(Q_h K_g^T / sqrt(d) + causal mask) V_g, g = h / (n_q / n_kv)
//
// Attention lives in attention_tc.cuh (fifth-generation tensor cores).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace serq {

// In-place rotate-half RoPE on heads [0, n_heads) of a token-major bf16 matrix
// (row stride ld elements): one thread per (token, head, pair).
__global__ void rope_kernel(__nv_bfloat16* __restrict__ x, int M, int ld, int n_heads, int head_dim, float log2_base,
                            int pos0) {
    const int half = head_dim >> 1;
    const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<size_t>(M) * n_heads * half) return;
    const int i = static_cast<int>(idx % half);
    const size_t t = idx / half;
    const int hd = static_cast<int>(t % n_heads);
    const int m = static_cast<int>(t / n_heads);
    const float inv_freq = exp2f(-(2.0f * static_cast<float>(i) / static_cast<float>(head_dim)) * log2_base);
    float sn, cs;
    sincosf(static_cast<float>(pos0 + m) * inv_freq, &sn, &cs);
    __nv_bfloat16* p = x + static_cast<size_t>(m) * ld + static_cast<size_t>(hd) * head_dim;
    const float a = __bfloat162float(p[i]), b = __bfloat162float(p[i + half]);
    p[i] = __float2bfloat16_rn(a * cs - b * sn);
    p[i + half] = __float2bfloat16_rn(b * cs + a * sn);
}

// out = bf16(a + b), eight bf16 per thread.
__global__ void add_bf16_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b, uint4* __restrict__ out,
                                size_t n8) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const uint4 x = a[i], y = b[i];
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(xs[e] << 16) + __uint_as_float(ys[e] << 16);
        const float hi = __uint_as_float(xs[e] & 0xFFFF0000u) + __uint_as_float(ys[e] & 0xFFFF0000u);
        r[e] = pack_bf16x2(lo, hi);
    }
    out[i] = make_uint4(r[0], r[1], r[2], r[3]);
}

}  // namespace serq
