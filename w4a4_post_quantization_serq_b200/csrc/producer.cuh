// Producers of a SERQ linear's input with the offline fold and the activation
// quantization fused into one pass over HBM.
//
// SERQ folds the saliency permutation and 1/s into the layer that produces
// the linear's input (reading notes Stage 3; gist.science/zh 2.3), so that
// layer can emit X^ = X diag(s)^-1 P^T directly. In a LLaMA block the
// producers are RMSNorm (input of q/k/v and of gate/up) and SwiGLU (input of
// down). These kernels compute each X^ row on the fly and hand it, eight
// values at a time, to the serq_quant_act row quantizers: one read of the
// producer's input, one write of the packed codes and scales, no bf16 X^ in
// HBM (an optional debug copy of X^ aside).
//
//   RMSNorm: rstd[m] = 1 / sqrt(fp32(sum_j H[m,j]^2) / K + eps)
//            X^[m,i] = bf16(fp32(H[m, perm[i]] * rstd[m]) * fp32(gamma[perm[i]] * inv_s[i]))
//   SwiGLU : X^[m,i] = bf16(fp32(fp32(silu(g) * u) * inv_s[i])),
//            g = Y[m, perm[i]], u = Y[m, F + perm[i]], silu(g) = g / (1 + exp(-g))
//
// Every step is one IEEE fp32 operation with round to nearest (no
// contraction). The sum of squares is accumulated in fp64 over the row
// (each square of a bf16 value is exact in fp64) and rounded once to fp32.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "quant_act.cuh"

namespace serq {

// Copy a row of `nchunk` 16-byte chunks to shared memory; returns this
// thread's fp64 sum of squares of the bf16 values it copied (if `squares`).
__device__ __forceinline__ double stage_row(const uint4* __restrict__ src, int nchunk, uint4* dst, bool squares) {
    double ss = 0.0;
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
        const uint4 v = __ldg(src + c);
        dst[c] = v;
        if (squares) {
            float f[8];
            bf16x8_to_f32(v, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += static_cast<double>(f[e]) * static_cast<double>(f[e]);
        }
    }
    return ss;
}

// Sum of a double over the CTA (kQuantThreads threads), fixed tree order.
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kQuantThreads / 32; ++w) t += red[w];
    return t;
}

// Eight consecutive positions 8c..8c+7 of the permutation and of 1/s[perm].
struct PermChunk {
    int j[8];
    float inv[8];
    __device__ __forceinline__ PermChunk(const int* __restrict__ perm, const float* __restrict__ inv_s, int c) {
        const int4 p0 = __ldg(reinterpret_cast<const int4*>(perm) + 2 * c);
        const int4 p1 = __ldg(reinterpret_cast<const int4*>(perm) + 2 * c + 1);
        const float4 i0 = __ldg(reinterpret_cast<const float4*>(inv_s) + 2 * c);
        const float4 i1 = __ldg(reinterpret_cast<const float4*>(inv_s) + 2 * c + 1);
        j[0] = p0.x; j[1] = p0.y; j[2] = p0.z; j[3] = p0.w;
        j[4] = p1.x; j[5] = p1.y; j[6] = p1.z; j[7] = p1.w;
        inv[0] = i0.x; inv[1] = i0.y; inv[2] = i0.z; inv[3] = i0.w;
        inv[4] = i1.x; inv[5] = i1.y; inv[6] = i1.z; inv[7] = i1.w;
    }
};

__device__ __forceinline__ uint4 pack_bf16x8(const float (&v)[8]) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}

// X^ chunk of the RMSNorm producer (row staged in shared memory, original order).
struct SrcRmsNorm {
    const __nv_bfloat16* h;
    const int* perm;
    const float* inv_s;
    const __nv_bfloat16* gamma;
    float rstd;
    uint4* xhat;  // NULL, or this row of the debug copy of X^
    __device__ __forceinline__ uint4 chunk(int c) const {
        const PermChunk pc(perm, inv_s, c);
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = pc.j[e];
            const float t = __fmul_rn(__bfloat162float(h[j]), rstd);
            const float g = __fmul_rn(__bfloat162float(__ldg(gamma + j)), pc.inv[e]);
            v[e] = __fmul_rn(t, g);
        }
        const uint4 out = pack_bf16x8(v);
        if (xhat != nullptr) xhat[c] = out;
        return out;
    }
};

// X^ chunk of the SwiGLU producer (the row [gate | up] staged in shared memory).
struct SrcSwiGlu {
    const __nv_bfloat16* y;
    int F;
    const int* perm;
    const float* inv_s;
    uint4* xhat;
    __device__ __forceinline__ uint4 chunk(int c) const {
        const PermChunk pc(perm, inv_s, c);
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = pc.j[e];
            const float g = __bfloat162float(y[j]);
            const float u = __bfloat162float(y[F + j]);
            const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
            v[e] = __fmul_rn(__fmul_rn(silu, u), pc.inv[e]);
        }
        const uint4 out = pack_bf16x8(v);
        if (xhat != nullptr) xhat[c] = out;
        return out;
    }
};

// X^ chunk of the plain fold (serq_fold_producer's arithmetic) of a row staged
// in shared memory: X^[m,i] = bf16(X[m, perm[i]] / s[perm[i]]).
struct SrcFold {
    const __nv_bfloat16* x;
    const int* perm;
    const float* s_perm;
    uint4* xhat;
    __device__ __forceinline__ uint4 chunk(int c) const {
        const PermChunk pc(perm, s_perm, c);  // .inv holds s[perm[i]] here
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __fdiv_rn(__bfloat162float(x[pc.j[e]]), pc.inv[e]);
        const uint4 out = pack_bf16x8(v);
        if (xhat != nullptr) xhat[c] = out;
        return out;
    }
};

struct ProducerParams {
    int K, r, rp;            // the consuming linear's input width, rank, padded rank
    const int* perm;         // [K] permuted position -> producer channel
    const float* inv_s;      // [K] 1 / s[perm[i]]
    const float* s_perm;     // [K] s[perm[i]] (the plain fold divides by it)
    const __nv_bfloat16* gamma;  // RMSNorm weight [K] (original order)
    float eps;
    void* xq;
    void* xs;
    void* xsq;
    void* xss;
    __nv_bfloat16* xhat;     // NULL or debug copy of X^ [M][K]
};

// Hand a row of X^ to the quantizer of the consumer's format (0 INT4, 1 MXFP4,
// 2 W4A8's INT8 activations).
template <int FMT, int MAXC, class Src>
__device__ __forceinline__ void quant_row(const Src& src, int m, int K, const ProducerParams& p, float* red) {
    if constexpr (FMT == 0)
        quant_row_int4<MAXC>(src, m, K, p.r, p.rp, static_cast<uint32_t*>(p.xq), static_cast<float*>(p.xs),
                             static_cast<uint32_t*>(p.xsq), static_cast<float*>(p.xss), red);
    else if constexpr (FMT == 1)
        quant_row_mxfp4(src, m, K, p.r, p.rp, static_cast<uint32_t*>(p.xq), static_cast<uint8_t*>(p.xs),
                        static_cast<uint32_t*>(p.xsq), static_cast<uint8_t*>(p.xss));
    else
        quant_row_int8<MAXC>(src, m, K, p.r, p.rp, static_cast<uint8_t*>(p.xq), static_cast<float*>(p.xs),
                             static_cast<uint8_t*>(p.xsq), static_cast<float*>(p.xss), red);
}

// One CTA per token row. kind 0: RMSNorm of H (M x K); kind 1: SwiGLU of Y (M x 2K);
// kind 2: the plain fold of X (M x K) (a producer that cannot fold itself).
// fmt 0: INT4, 2: INT8 (MAXC chunks per thread), 1: MXFP4.
// Several CTAs per SM: a row is a short job (one read of the row, its
// quantization), so the SM needs several rows in flight to hide the latency.
// MXFP4 rows hold nothing across the row (4 CTAs per SM); the per-token
// integer formats keep the row's chunks in registers (MAXC of them).
template <int KIND, int FMT, int MAXC>
__global__ void __launch_bounds__(kQuantThreads, FMT == 1 ? 4 : (MAXC > 8 ? 2 : 3))
producer_quant_kernel(const uint4* __restrict__ in, const ProducerParams p) {
    extern __shared__ __align__(16) uint8_t smem_prod[];
    __shared__ double red64[kQuantThreads / 32];
    __shared__ float red[64];
    pdl_launch_dependents();
    const int m = blockIdx.x;
    const int K = p.K;
    uint4* row = reinterpret_cast<uint4*>(smem_prod);
    uint4* xhat_row = p.xhat != nullptr ? reinterpret_cast<uint4*>(p.xhat + static_cast<size_t>(m) * K) : nullptr;
    if constexpr (KIND == 0) {
        const double part = stage_row(in + static_cast<size_t>(m) * (K >> 3), K >> 3, row, true);
        const double ss = block_sum_f64(part, red64);
        const float ms = __fdiv_rn(__double2float_rn(ss), static_cast<float>(K));
        const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
        const SrcRmsNorm src{reinterpret_cast<const __nv_bfloat16*>(row), p.perm, p.inv_s, p.gamma, rstd, xhat_row};
        quant_row<FMT, MAXC>(src, m, K, p, red);
    } else if constexpr (KIND == 2) {
        stage_row(in + static_cast<size_t>(m) * (K >> 3), K >> 3, row, false);
        __syncthreads();
        const SrcFold src{reinterpret_cast<const __nv_bfloat16*>(row), p.perm, p.s_perm, xhat_row};
        quant_row<FMT, MAXC>(src, m, K, p, red);
    } else {
        stage_row(in + static_cast<size_t>(m) * (K >> 2), K >> 2, row, false);
        __syncthreads();
        const SrcSwiGlu src{reinterpret_cast<const __nv_bfloat16*>(row), K, p.perm, p.inv_s, xhat_row};
        quant_row<FMT, MAXC>(src, m, K, p, red);
    }
}

}  // namespace serq
