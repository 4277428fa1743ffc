// The LLaMA block around the SERQ linears, for the time-to-first-token of a
// 2K-token prefill (the measurement the reading notes report under
// "GPU 性能分析"): rotary position embedding, causal grouped-query attention
// in bf16, and the residual add. The pages do not restate these layers; they
// follow the standard LLaMA definitions:
//   RoPE (rotate-half): for pair i < d/2 of a head at position p,
//       angle = p * base^(-2i/d), (x_i, x_{i+d/2}) <- (x_i c - x_{i+d/2} s, x_{i+d/2} c + x_i s)
//   attention: O_h = softmax(Q_h K_g^T / sqrt(d) + causal mask) V_g, g = h / (n_q / n_kv)
//
// Attention is a flash-attention style kernel on the warp-level bf16 tensor
// core instruction (mma.sync m16n8k16, fp32 accumulation): 64 queries of one
// head per CTA (16 per warp), 64-key tiles of K and V double-buffered in
// shared memory by cp.async (128-byte rows swizzled by XOR of the 16-byte
// chunk with the row), scores and the running softmax kept in registers.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace serq {
namespace att {

constexpr int D = 128;        // head dimension
constexpr int BM = 64;        // queries per CTA
constexpr int BN = 64;        // keys per tile
constexpr int THREADS = 128;  // 4 warps x 16 query rows
constexpr int TILE_BYTES = 64 * D * 2;                  // 16 KB
constexpr int SMEM_BYTES = TILE_BYTES * 5 + 128;        // Q, 2 x K, 2 x V

}  // namespace att

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of the 16-byte chunk c (8 dims) of row r in a swizzled 64 x 128 bf16 tile.
__device__ __forceinline__ uint32_t att_off(int r, int c) {
    return static_cast<uint32_t>(r * 256 + ((c ^ (r & 7)) << 4));
}

// Copy rows [row0, row0 + 64) of a token-major matrix (leading dimension ld
// elements, this head's 128 columns at col0) into a swizzled tile; rows at or
// past M read as zeros.
__device__ __forceinline__ void att_load_tile(uint32_t dst, const __nv_bfloat16* __restrict__ base, int ld, int col0,
                                              int row0, int M) {
    for (int t = threadIdx.x; t < 64 * 16; t += att::THREADS) {
        const int r = t >> 4, c = t & 15;
        const int row = row0 + r;
        const bool ok = row < M;
        const __nv_bfloat16* src = base + static_cast<size_t>(ok ? row : 0) * ld + col0 + c * 8;
        cp_async16(dst + att_off(r, c), src, ok);
    }
}

// grid (ceil(M / 64), n_q): CTA (qb, h) computes queries [64 qb, +64) of head h.
// Blocks are taken last-first so the longest (most keys) start first.
__global__ void __launch_bounds__(att::THREADS)
attention_prefill_kernel(const __nv_bfloat16* __restrict__ q, int ldq, const __nv_bfloat16* __restrict__ k,
                         const __nv_bfloat16* __restrict__ v, int ldkv, int M, int n_q, int n_kv,
                         float scale_log2, __nv_bfloat16* __restrict__ o, int ldo) {
    using namespace att;
    extern __shared__ __align__(128) uint8_t smem_att[];
    const uint32_t sQ = smem_u32(smem_att);
    const uint32_t sK0 = sQ + TILE_BYTES;
    const uint32_t sV0 = sK0 + 2 * TILE_BYTES;
    const int qb = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);
    const int h = blockIdx.y;
    const int g = h / (n_q / n_kv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = qb * BM;
    const int n_tiles = qb + 1;  // causal: key tiles 0 .. qb (BM == BN)

    att_load_tile(sQ, q, ldq, h * D, q0, M);
    att_load_tile(sK0, k, ldkv, g * D, 0, M);
    att_load_tile(sV0, v, ldkv, g * D, 0, M);
    cp_async_commit();

    uint32_t qf[8][4];
    float acc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};
    const int qrow = q0 + warp * 16 + (lane >> 2);  // this thread's rows: qrow and qrow + 8

    for (int j = 0; j < n_tiles; ++j) {
        const int buf = j & 1;
        if (j + 1 < n_tiles) {
            att_load_tile(sK0 + (buf ^ 1) * TILE_BYTES, k, ldkv, g * D, (j + 1) * BN, M);
            att_load_tile(sV0 + (buf ^ 1) * TILE_BYTES, v, ldkv, g * D, (j + 1) * BN, M);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (j == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int c = 2 * kk + (lane >> 4);
                ldsm_x4(sQ + att_off(r, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
            }
        }
        const uint32_t sK = sK0 + buf * TILE_BYTES;
        const uint32_t sV = sV0 + buf * TILE_BYTES;
        // S = Q K^T for 16 queries x 64 keys
        float s[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {  // pairs of 8-key tiles
                const int key = np * 16 + (lane & 7) + 8 * (lane >> 4);
                const int c = 2 * kk + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sK + att_off(key, c), b0, b1, b2, b3);
                mma_bf16_16816(s[2 * np], qf[kk], b0, b1);
                mma_bf16_16816(s[2 * np + 1], qf[kk], b2, b3);
            }
        }
        // causal mask on the diagonal tile, then the running softmax (log2 domain)
        float p_max[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int row = qrow + ((e >> 1) << 3);
                const int key = j * BN + nt * 8 + ((lane & 3) << 1) + (e & 1);
                float t = s[nt][e] * scale_log2;
                if (j == qb && key > row) t = -INFINITY;
                s[nt][e] = t;
                p_max[e >> 1] = fmaxf(p_max[e >> 1], t);
            }
        }
        float corr[2];
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            p_max[sl] = fmaxf(p_max[sl], __shfl_xor_sync(0xFFFFFFFFu, p_max[sl], 1));
            p_max[sl] = fmaxf(p_max[sl], __shfl_xor_sync(0xFFFFFFFFu, p_max[sl], 2));
            const float m_new = fmaxf(m_run[sl], p_max[sl]);
            corr[sl] = exp2f(m_run[sl] - m_new);  // 0 on the first tile (m_run = -inf)
            m_run[sl] = m_new;
            l_run[sl] *= corr[sl];
        }
        uint32_t pf[4][4];  // P as bf16 A fragments, one per 16-key step
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                p[e] = exp2f(s[nt][e] - m_run[e >> 1]);
                l_run[e >> 1] += p[e];
            }
            const int ks = nt >> 1, hi = nt & 1;
            pf[ks][2 * hi] = pack_bf16x2(p[0], p[1]);
            pf[ks][2 * hi + 1] = pack_bf16x2(p[2], p[3]);
        }
#pragma unroll
        for (int dt = 0; dt < 16; ++dt) {
            acc[dt][0] *= corr[0];
            acc[dt][1] *= corr[0];
            acc[dt][2] *= corr[1];
            acc[dt][3] *= corr[1];
        }
        // O += P V (V tile keys x dims, read transposed)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-dim tiles
                const int key = ks * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int c = 2 * dp + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sV + att_off(key, c), b0, b1, b2, b3);
                mma_bf16_16816(acc[2 * dp], pf[ks], b0, b1);
                mma_bf16_16816(acc[2 * dp + 1], pf[ks], b2, b3);
            }
        }
        __syncthreads();  // this buffer is reloaded two tiles later
    }
    cp_async_wait<0>();
    // normalise and store: thread holds rows qrow, qrow + 8, dims 8 dt + 2 (lane & 3)
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
        l_run[sl] += __shfl_xor_sync(0xFFFFFFFFu, l_run[sl], 1);
        l_run[sl] += __shfl_xor_sync(0xFFFFFFFFu, l_run[sl], 2);
    }
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
        const int row = qrow + 8 * sl;
        if (row >= M) continue;
        const float inv = 1.0f / l_run[sl];
        __nv_bfloat16* dst = o + static_cast<size_t>(row) * ldo + h * D + ((lane & 3) << 1);
#pragma unroll
        for (int dt = 0; dt < 16; ++dt)
            *reinterpret_cast<uint32_t*>(dst + dt * 8) = pack_bf16x2(acc[dt][2 * sl] * inv, acc[dt][2 * sl + 1] * inv);
    }
}

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
