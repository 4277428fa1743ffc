// serq_prepare kernels (offline; reading notes Stage 1-3, gist.science/zh 2.1-2.3).
//
//   a_j  = max_t |X[t, j]|                         (calibration)
//   s_j  = sqrt(a_j / max_n |W[j, n]|), 1 if either is 0      (Stage 1, SAF)
//   perm = channels by s descending, ties by index             (Stage 2)
//   W^[i, n] = fp32(s[perm[i]] * W[perm[i], n])                (Stage 2)
//   W^_q: INT4 per output channel over K, or MXFP4 per 32 along K (RTN)
//   R = W^[:r] - deq(W^_q)[:r]; Q(R): INT4 per output channel / MXFP4 per 32
//
// All arithmetic is IEEE fp32 with explicit single roundings, so the packed
// results are reproducible bit for bit by a scalar restatement.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "quant_act.cuh"

namespace serq {

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}

// a_j = max_t |X[t, j]| via an atomic max on the (non-negative) float bits.
__global__ void calib_absmax_kernel(const __nv_bfloat16* __restrict__ X, int M, int K, int rows_per_cta,
                                    unsigned int* __restrict__ out_bits) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    const int t0 = blockIdx.y * rows_per_cta;
    const int t1 = min(M, t0 + rows_per_cta);
    float a = 0.0f;
    for (int t = t0; t < t1; ++t) a = fmaxf(a, fabsf(bf16_at(X, static_cast<size_t>(t) * K + j)));
    atomicMax(out_bits + j, __float_as_uint(a));
}

// b_j = max_n |W[j, n]|, one warp per row j.
__global__ void row_absmax_kernel(const __nv_bfloat16* __restrict__ W, int K, int N, float* __restrict__ b) {
    const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (j >= K) return;
    const uint4* rowp = reinterpret_cast<const uint4*>(W + static_cast<size_t>(j) * N);
    float a = 0.0f;
    for (int c = lane; c < N / 8; c += 32) {
        float f[8];
        bf16x8_to_f32(__ldg(rowp + c), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(f[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    if (lane == 0) b[j] = a;
}

__global__ void saf_scale_kernel(const float* __restrict__ a, const float* __restrict__ b, int K,
                                 float* __restrict__ s) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    const float aj = a[j], bj = b[j];
    s[j] = (aj > 0.0f && bj > 0.0f) ? __fsqrt_rn(__fdiv_rn(aj, bj)) : 1.0f;
}

// rank of channel j in the order "s descending, lower index first on ties";
// perm[rank] = j, s_perm[rank] = s_j, inv_s[rank] = 1 / s_j.
__global__ void saliency_rank_kernel(const float* __restrict__ s, int K, int* __restrict__ perm,
                                     float* __restrict__ s_perm, float* __restrict__ inv_s) {
    __shared__ float tile[1024];
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const float sj = j < K ? s[j] : 0.0f;
    int rank = 0;
    for (int base = 0; base < K; base += 1024) {
        const int n = min(1024, K - base);
        __syncthreads();
        for (int t = threadIdx.x; t < n; t += blockDim.x) tile[t] = s[base + t];
        __syncthreads();
        if (j < K) {
            for (int t = 0; t < n; ++t) {
                const float si = tile[t];
                const int i = base + t;
                rank += (si > sj) || (si == sj && i < j);
            }
        }
    }
    if (j < K) {
        perm[rank] = j;
        s_perm[rank] = sj;
        inv_s[rank] = __fdiv_rn(1.0f, sj);
    }
}

// Column absmax of W^ over all K rows (INT4 per-output-channel scale).
// The absmax is permutation-invariant, so rows are visited in original order.
__global__ void weight_colamax_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ s, int K,
                                      int N, int rows_per_cta, unsigned int* __restrict__ out_bits) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const int j0 = blockIdx.y * rows_per_cta;
    const int j1 = min(K, j0 + rows_per_cta);
    float a = 0.0f;
    for (int j = j0; j < j1; ++j) a = fmaxf(a, fabsf(__fmul_rn(s[j], bf16_at(W, static_cast<size_t>(j) * N + n))));
    atomicMax(out_bits + n, __float_as_uint(a));
}

__device__ __forceinline__ float what_at(const __nv_bfloat16* W, const int* perm, const float* s_perm, int N,
                                         int i, int n) {
    return __fmul_rn(s_perm[i], bf16_at(W, static_cast<size_t>(perm[i]) * N + n));
}

// W^_q (INT4): thread (n, 32-row block b of permuted rows) -> 16 packed bytes.
__global__ void weight_quant_int4_kernel(const __nv_bfloat16* __restrict__ W, const int* __restrict__ perm,
                                         const float* __restrict__ s_perm,
                                         const unsigned int* __restrict__ colamax_bits, int K, int N,
                                         uint8_t* __restrict__ wq, float* __restrict__ sw) {
    const int n = blockIdx.x * 32 + threadIdx.x;
    const int b = blockIdx.y * blockDim.y + threadIdx.y;
    if (n >= N || b * 32 >= K) return;
    const float scale = __fdiv_rn(__uint_as_float(colamax_bits[n]), 7.0f);
    if (b == 0) sw[n] = scale;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll 8
    for (int e = 0; e < 32; ++e) {
        const float v = what_at(W, perm, s_perm, N, b * 32 + e, n);
        w[e >> 3] |= int4_code(v, scale) << (4 * (e & 7));
    }
    *reinterpret_cast<uint4*>(wq + static_cast<size_t>(n) * (K / 2) + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
}

// W^_q (MXFP4): thread (n, block b) -> 16 packed bytes + one E8M0 byte.
__global__ void weight_quant_mxfp4_kernel(const __nv_bfloat16* __restrict__ W, const int* __restrict__ perm,
                                          const float* __restrict__ s_perm, int K, int N,
                                          uint8_t* __restrict__ wq, uint8_t* __restrict__ w_atoms) {
    const int n = blockIdx.x * 32 + threadIdx.x;
    const int b = blockIdx.y * blockDim.y + threadIdx.y;
    if (n >= N || b * 32 >= K) return;
    float v[32];
    float a = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        v[e] = what_at(W, perm, s_perm, N, b * 32 + e, n);
        a = fmaxf(a, fabsf(v[e]));
    }
    const int E = mx_exponent(a);
    const float inv = mx_inv_scale(E);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float g[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = __fmul_rn(v[q * 8 + e], inv);
        w[q] = e2m1x8(g);
    }
    *reinterpret_cast<uint4*>(wq + static_cast<size_t>(n) * (K / 2) + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    w_atoms[sf_atom_offset(n, b, K / 128)] = static_cast<uint8_t>(E + 127);
}

// Residual, INT4: thread per output channel n.
//   R[i, n] = fp32(W^[i, n] - fp32(q_w[i, n] * s_w[n])),  i < r
//   s_R[n] = fp32(max_i |R| / 7),  Q(R) = clip(rne(R / s_R))
__global__ void residual_int4_kernel(const __nv_bfloat16* __restrict__ W, const int* __restrict__ perm,
                                     const float* __restrict__ s_perm, const float* __restrict__ sw, int N, int r,
                                     int rp, uint8_t* __restrict__ rq, float* __restrict__ sR) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const float swn = sw[n];
    float a = 0.0f;
    for (int i = 0; i < r; ++i) {
        const float v = what_at(W, perm, s_perm, N, i, n);
        const int q = static_cast<int>(int4_code(v, swn) << 28) >> 28;
        a = fmaxf(a, fabsf(__fsub_rn(v, __fmul_rn(static_cast<float>(q), swn))));
    }
    const float srn = __fdiv_rn(a, 7.0f);
    sR[n] = srn;
    for (int b = 0; b < rp / 32; ++b) {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        for (int e = 0; e < 32; ++e) {
            const int i = b * 32 + e;
            if (i < r) {
                const float v = what_at(W, perm, s_perm, N, i, n);
                const int q = static_cast<int>(int4_code(v, swn) << 28) >> 28;
                const float R = __fsub_rn(v, __fmul_rn(static_cast<float>(q), swn));
                w[e >> 3] |= int4_code(R, srn) << (4 * (e & 7));
            }
        }
        *reinterpret_cast<uint4*>(rq + static_cast<size_t>(n) * (rp / 2) + b * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// E2M1 code -> value. Twice the magnitudes {0,.5,1,1.5,2,3,4,6} are the
// nibbles of 0xC8643210.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
    const float v = static_cast<float>((0xC8643210u >> (4u * (code & 7u))) & 0xFu) * 0.5f;
    return (code & 8u) ? -v : v;
}

// 2^E for E in [-127, 125] (2^-127 is a subnormal).
__device__ __forceinline__ float exp2_int(int E) {
    return E >= -126 ? __uint_as_float(static_cast<uint32_t>(E + 127) << 23) : __uint_as_float(0x00400000u);
}

// Residual, MXFP4: thread (n, 32-row block b of the first rp rows).
// The main weight block b covers the same rows, so its exponent is recomputed
// from all 32 rows; R is taken on rows i < r and quantized in its own block.
__global__ void residual_mxfp4_kernel(const __nv_bfloat16* __restrict__ W, const int* __restrict__ perm,
                                      const float* __restrict__ s_perm, int K, int N, int r, int rp,
                                      uint8_t* __restrict__ rq, uint8_t* __restrict__ r_atoms) {
    const int n = blockIdx.x * 32 + threadIdx.x;
    const int b = blockIdx.y * blockDim.y + threadIdx.y;
    if (n >= N || b * 32 >= rp) return;
    float v[32];
    float a = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int i = b * 32 + e;
        v[e] = i < K ? what_at(W, perm, s_perm, N, i, n) : 0.0f;
        a = fmaxf(a, fabsf(v[e]));
    }
    const int Ew = mx_exponent(a);
    const float inv_w = mx_inv_scale(Ew);
    const float unit_w = exp2_int(Ew);
    float ra = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float g[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = __fmul_rn(v[q * 8 + e], inv_w);
        const uint32_t codes = e2m1x8(g);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int i = b * 32 + q * 8 + e;
            const float deq = __fmul_rn(e2m1_value((codes >> (4 * e)) & 0xFu), unit_w);
            v[q * 8 + e] = (i < r) ? __fsub_rn(v[q * 8 + e], deq) : 0.0f;
            ra = fmaxf(ra, fabsf(v[q * 8 + e]));
        }
    }
    const int Er = mx_exponent(ra);
    const float inv_r = mx_inv_scale(Er);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float g[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = __fmul_rn(v[q * 8 + e], inv_r);
        w[q] = e2m1x8(g);
    }
    *reinterpret_cast<uint4*>(rq + static_cast<size_t>(n) * (rp / 2) + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    r_atoms[sf_atom_offset(n, b, (rp / 32 + 3) / 4)] = static_cast<uint8_t>(Er + 127);
}

// Residual slot holding a given matrix G (r x N, bf16, row-major) instead of
// W~_s - Q(W~_s): the second factor of the two-factor baseline (L2QER's L2).
// Quantized exactly as Q(R) is.
//   INT4 : thread per output channel n: s[n] = fp32(max_i |G[i, n]| / 7), codes rne(G / s)
__global__ void given_residual_int4_kernel(const __nv_bfloat16* __restrict__ G, int N, int r, int rp,
                                           uint8_t* __restrict__ rq, float* __restrict__ sR) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float a = 0.0f;
    for (int i = 0; i < r; ++i) a = fmaxf(a, fabsf(bf16_at(G, static_cast<size_t>(i) * N + n)));
    const float srn = __fdiv_rn(a, 7.0f);
    sR[n] = srn;
    for (int b = 0; b < rp / 32; ++b) {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        for (int e = 0; e < 32; ++e) {
            const int i = b * 32 + e;
            if (i < r) w[e >> 3] |= int4_code(bf16_at(G, static_cast<size_t>(i) * N + n), srn) << (4 * (e & 7));
        }
        *reinterpret_cast<uint4*>(rq + static_cast<size_t>(n) * (rp / 2) + b * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

//   MXFP4: thread (n, 32-row block b along r): E8M0 exponent of the block, E2M1 codes
__global__ void given_residual_mxfp4_kernel(const __nv_bfloat16* __restrict__ G, int N, int r, int rp,
                                            uint8_t* __restrict__ rq, uint8_t* __restrict__ r_atoms) {
    const int n = blockIdx.x * 32 + threadIdx.x;
    const int b = blockIdx.y * blockDim.y + threadIdx.y;
    if (n >= N || b * 32 >= rp) return;
    float v[32];
    float a = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int i = b * 32 + e;
        v[e] = i < r ? bf16_at(G, static_cast<size_t>(i) * N + n) : 0.0f;
        a = fmaxf(a, fabsf(v[e]));
    }
    const int E = mx_exponent(a);
    const float inv = mx_inv_scale(E);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float g[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = __fmul_rn(v[q * 8 + e], inv);
        w[q] = e2m1x8(g);
    }
    *reinterpret_cast<uint4*>(rq + static_cast<size_t>(n) * (rp / 2) + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    // blocks past the last real one stay zero (padding)
    if (b * 32 < r) r_atoms[sf_atom_offset(n, b, (rp / 32 + 3) / 4)] = static_cast<uint8_t>(E + 127);
}

// Output columns of a gate/up weight [W_gate | W_up] (K x 2F) arranged for the
// SwiGLU epilogue of the down linear it feeds (Stage 3: the down linear's
// input permutation merged into the producer's weight): column block t
// (256 wide) holds the gate then the up columns of down's permuted input
// positions 128 t .. 128 t + 127:
//   Wp[k][256 t + c]       = W[k][perm_d[128 t + c]]
//   Wp[k][256 t + 128 + c] = W[k][F + perm_d[128 t + c]]
__global__ void swiglu_arrange_kernel(const __nv_bfloat16* __restrict__ W, int K, int F, const int* __restrict__ perm_d,
                                      __nv_bfloat16* __restrict__ Wp) {
    const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t cols = 2 * static_cast<size_t>(F);
    if (idx >= static_cast<size_t>(K) * cols) return;
    const size_t k = idx / cols;
    const int col = static_cast<int>(idx - k * cols);
    const int t = col >> 8, c = col & 255;
    const int src = c < 128 ? perm_d[128 * t + c] : F + perm_d[128 * t + c - 128];
    Wp[idx] = W[k * cols + src];
}

// dst[row][i] = bf16(src[row][perm[i]] / s[perm[i]])  (Stage 3 producer fold)
__global__ void fold_producer_kernel(const __nv_bfloat16* __restrict__ src, int rows, int K,
                                     const int* __restrict__ perm, const float* __restrict__ s_perm,
                                     __nv_bfloat16* __restrict__ dst) {
    const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<size_t>(rows) * K) return;
    const int i = static_cast<int>(idx % K);
    const size_t row = idx / K;
    const float x = bf16_at(src, row * K + perm[i]);
    dst[idx] = __float2bfloat16_rn(__fdiv_rn(x, s_perm[i]));
}

// Wide scale layout of the CTA-pair kernel: for each pair of 128-row blocks
// (2p, 2p+1) and scale atom j, a 4 KB piece read by one tcgen05.cp .128x256b
// as 128 rows x 32 bytes in 8-row x 16-byte core matrices (row group g at
// 256 g, its two column halves 128 bytes apart). Row l must hold row l % 32 of
// atom (2p, j) in its first half and of atom (2p+1, j) in its second, which is
// what two .32x128b.warpx4 copies of the two atoms would put in the same 8
// tensor-memory columns; so row group g, half h holds bytes [128 (g % 4),
// +128) of atom (2p+h, j) (a missing odd block reads as zeros). One thread
// per 16 bytes.
__global__ void scale_widen_kernel(const uint8_t* __restrict__ atoms, int row_blocks, int atoms_k,
                                   uint8_t* __restrict__ wide, size_t wide_bytes) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // 16-byte unit
    if (i * 16 >= wide_bytes) return;
    const size_t piece = i / 256;                  // 4 KB pieces
    const int within = static_cast<int>(i % 256);  // 16-byte units in the piece
    const int group = within / 16;                 // 8-row group (256 bytes)
    const int half = (within / 8) % 2;             // even / odd row block
    const int row = within % 8;                    // row within the core matrix
    const int j = static_cast<int>(piece % atoms_k);
    const int pair = static_cast<int>(piece / atoms_k);
    const int rb = 2 * pair + half;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (rb < row_blocks)
        v = reinterpret_cast<const uint4*>(atoms + (static_cast<size_t>(rb) * atoms_k + j) * 512)[8 * (group % 4) + row];
    reinterpret_cast<uint4*>(wide)[i] = v;
}

}  // namespace serq
