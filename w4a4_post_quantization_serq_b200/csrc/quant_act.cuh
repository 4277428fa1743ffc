// serq_quant_act kernels: per-token activation quantization and the salient
// slice X~_s = X^[:, :r] under its own scale.
//
// INT4  ("基础量化", reading notes): s = max|x| / 7, q = clip(rne(x / s), -7, 7),
//       one fp32 scale per token; the slice uses the absmax of its r columns.
// MXFP4 (OCP MX v1.0, named by the pages as MXFP4): per 32-element block,
//       E = floor(log2 amax) - 2 (clamped to [-127, 127]), codes = E2M1
//       round-to-nearest-even of x * 2^-E (saturating at 6).
//
// Every quantization decision is made in IEEE fp32 with one rounding per
// operation (explicit __fdiv_rn; no contraction), so the codes match a
// scalar fp32 restatement bit for bit.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace serq {

constexpr int kQuantThreads = 256;
constexpr int kInt4Max = 7;     // INT4 activation codes: s = max|x| / 7
constexpr int kInt8Max = 127;   // INT8 (W4A8) activation codes: s = max|x| / 127

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// rint(fl(x / s)) (IEEE division, ties to even) for |x / s| <= 128, dividing
// only near a tie: q = fl(x * fl(1/s)) is within 2^-22 |x / s| (< 4e-5) of
// x / s, so when q is farther than 1e-4 from every half-integer (|q - rint(q)|
// < 0.4999), fl(x / s) lies on the same side of it and rounds to the same
// integer. (inv_s = inf or a NaN q fails the test and takes the division.)
__device__ __noinline__ float rint_div(float x, float s) { return rintf(__fdiv_rn(x, s)); }

__device__ __forceinline__ float rint_quot(float x, float s, float inv_s) {
    const float q = __fmul_rn(x, inv_s);
    const float r = rintf(q);
    if (fabsf(q - r) < 0.4999f) return r;
    return rint_div(x, s);  // rare: kept out of line
}

// INT4 code of x under scale s (two's complement nibble); 0 when s == 0.
// |x| <= the absmax s was taken from, so |x / s| <= 7 (1 + 2^-23).
__device__ __forceinline__ uint32_t int4_code(float x, float s, float inv_s) {
    if (!(s > 0.0f)) return 0u;
    float q = rint_quot(x, s, inv_s);
    q = fminf(fmaxf(q, -7.0f), 7.0f);
    return static_cast<uint32_t>(static_cast<int>(q)) & 0xFu;
}

// The same with the division always taken (the offline weight quantizers).
__device__ __forceinline__ uint32_t int4_code(float x, float s) {
    if (!(s > 0.0f)) return 0u;
    float q = rintf(__fdiv_rn(x, s));
    q = fminf(fmaxf(q, -7.0f), 7.0f);
    return static_cast<uint32_t>(static_cast<int>(q)) & 0xFu;
}

// Shared MX exponent of a block from its absmax: floor(log2 amax) - 2, read
// off the fp32 exponent field; zero and subnormal maxima give -127.
__device__ __forceinline__ int mx_exponent(float amax) {
    const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
    if (e == 0) return -127;
    const int E = e - 127 - 2;
    return E < -127 ? -127 : E;
}

// 2^-E for E in [-127, 125] (always a normal float).
__device__ __forceinline__ float mx_inv_scale(int E) {
    return __uint_as_float(static_cast<uint32_t>(127 - E) << 23);
}

// Eight already-scaled floats -> eight E2M1 codes packed in a 32-bit word,
// element 0 in the lowest nibble (round to nearest even, saturate to +-6).
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Byte offset of the scale of (row, block) in the tensor-core scale atom
// layout: 128 rows x 4 blocks per 512-byte atom, atoms ordered by row block
// then block group.
__device__ __forceinline__ size_t sf_atom_offset(int row, int blk, int atoms_per_rowblock) {
    return (static_cast<size_t>(row >> 7) * atoms_per_rowblock + (blk >> 2)) * 512u +
           static_cast<size_t>((row & 31) * 16 + ((row >> 5) & 3) * 4 + (blk & 3));
}

__device__ __forceinline__ float block_max2(float& a, float& b, float* red) {
    // reduce two maxima over the CTA; red holds 2 * (kQuantThreads / 32) floats
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        b = fmaxf(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[warp] = a;
        red[32 + warp] = b;
    }
    __syncthreads();
    a = red[0];
    b = red[32];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) {
        a = fmaxf(a, red[w]);
        b = fmaxf(b, red[32 + w]);
    }
    return a;
}

// ---------------------------------------------------------------- row quantizers
// A "chunk source" yields the row's values eight at a time as packed bf16
// (chunk c = positions 8c .. 8c+7 of X^[m, :]); the quantizers below turn a
// row into serq_quant_act's outputs. The plain quantizer reads X^ from global
// memory; the fused producers compute X^ on the fly (producer.cuh).
struct SrcBf16Row {
    const uint4* row;
    __device__ __forceinline__ uint4 chunk(int c) const { return __ldg(row + c); }
};

// INT4, one CTA per row. MAXC = 16-byte chunks held per thread (K <= 8 * 256 * MAXC).
template <int MAXC, class Src>
__device__ __forceinline__ void quant_row_int4(const Src& src, int m, int K, int r, int rp, uint32_t* __restrict__ xq,
                                               float* __restrict__ xs, uint32_t* __restrict__ xsq,
                                               float* __restrict__ xss, float* red) {
    const int nchunk = K >> 3;
    uint4 v[MAXC];
    float amax = 0.0f, amax_s = 0.0f;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
        const int c = threadIdx.x + j * kQuantThreads;
        if (c < nchunk) {
            v[j] = src.chunk(c);
            float f[8];
            bf16x8_to_f32(v[j], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = fabsf(f[e]);
                amax = fmaxf(amax, a);
                if (c * 8 + e < r) amax_s = fmaxf(amax_s, a);
            }
        }
    }
    block_max2(amax, amax_s, red);
    const float s = __fdiv_rn(amax, 7.0f);
    const float ss = __fdiv_rn(amax_s, 7.0f);
    const float inv = __fdiv_rn(1.0f, s), invs = __fdiv_rn(1.0f, ss);
    if (threadIdx.x == 0) {
        xs[m] = s;
        if (rp > 0) xss[m] = ss;
    }
    const int nchunk_s = rp >> 3;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
        const int c = threadIdx.x + j * kQuantThreads;
        if (c < nchunk) {
            float f[8];
            bf16x8_to_f32(v[j], f);
            uint32_t w = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) w |= int4_code(f[e], s, inv) << (4 * e);
            xq[static_cast<size_t>(m) * nchunk + c] = w;
            if (c < nchunk_s) {
                uint32_t ws = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (c * 8 + e < r) ws |= int4_code(f[e], ss, invs) << (4 * e);
                xsq[static_cast<size_t>(m) * nchunk_s + c] = ws;
            }
        }
    }
}

// INT8 code of x under scale s (the W4A8 activations): clip(rne(x / s), -127, 127)
// as a byte; 0 when s == 0.
__device__ __forceinline__ uint32_t int8_code(float x, float s, float inv_s) {
    if (!(s > 0.0f)) return 0u;
    float q = rint_quot(x, s, inv_s);
    q = fminf(fmaxf(q, -127.0f), 127.0f);
    return static_cast<uint32_t>(static_cast<int>(q)) & 0xFFu;
}

// INT8 (W4A8 activations), one CTA per row: s = max|x| / 127, one byte per code;
// the salient slice under the absmax of its r columns. Same structure as INT4.
template <int MAXC, class Src>
__device__ __forceinline__ void quant_row_int8(const Src& src, int m, int K, int r, int rp, uint8_t* __restrict__ xq,
                                               float* __restrict__ xs, uint8_t* __restrict__ xsq,
                                               float* __restrict__ xss, float* red) {
    const int nchunk = K >> 3;
    uint4 v[MAXC];
    float amax = 0.0f, amax_s = 0.0f;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
        const int c = threadIdx.x + j * kQuantThreads;
        if (c < nchunk) {
            v[j] = src.chunk(c);
            float f[8];
            bf16x8_to_f32(v[j], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = fabsf(f[e]);
                amax = fmaxf(amax, a);
                if (c * 8 + e < r) amax_s = fmaxf(amax_s, a);
            }
        }
    }
    block_max2(amax, amax_s, red);
    const float s = __fdiv_rn(amax, 127.0f);
    const float ss = __fdiv_rn(amax_s, 127.0f);
    const float inv = __fdiv_rn(1.0f, s), invs = __fdiv_rn(1.0f, ss);
    if (threadIdx.x == 0) {
        xs[m] = s;
        if (rp > 0) xss[m] = ss;
    }
    const int nchunk_s = rp >> 3;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
        const int c = threadIdx.x + j * kQuantThreads;
        if (c < nchunk) {
            float f[8];
            bf16x8_to_f32(v[j], f);
            uint32_t w0 = 0, w1 = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                w0 |= int8_code(f[e], s, inv) << (8 * e);
                w1 |= int8_code(f[4 + e], s, inv) << (8 * e);
            }
            *reinterpret_cast<uint2*>(xq + static_cast<size_t>(m) * K + c * 8) = make_uint2(w0, w1);
            if (c < nchunk_s) {
                uint32_t s0 = 0, s1 = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (c * 8 + e < r) s0 |= int8_code(f[e], ss, invs) << (8 * e);
                    if (c * 8 + 4 + e < r) s1 |= int8_code(f[4 + e], ss, invs) << (8 * e);
                }
                *reinterpret_cast<uint2*>(xsq + static_cast<size_t>(m) * rp + c * 8) = make_uint2(s0, s1);
            }
        }
    }
}

// One 16-byte chunk (eight values f, positions 8c..8c+7 of row m) of an MXFP4
// row: the block maximum over the four lanes that hold the block's chunks
// (all 32 lanes must call this together), E8M0 exponent, E2M1 codes, and the
// salient slice's own block inside the first rp columns. Nothing is written
// for an invalid chunk (its values must be zeros).
__device__ __forceinline__ void mx_chunk_out(const float (&f)[8], bool valid, int c, int m, int r, int rp, int nchunk,
                                             uint32_t* __restrict__ xq, uint8_t* __restrict__ xs_atoms,
                                             uint32_t* __restrict__ xsq, uint8_t* __restrict__ xss_atoms,
                                             int atoms_k, int atoms_s) {
    const int nchunk_s = rp >> 3;
    float a = 0.0f, as = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        a = fmaxf(a, fabsf(f[e]));
        if (c * 8 + e < r) as = fmaxf(as, fabsf(f[e]));
    }
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
    as = fmaxf(as, __shfl_xor_sync(0xFFFFFFFFu, as, 1));
    as = fmaxf(as, __shfl_xor_sync(0xFFFFFFFFu, as, 2));
    if (!valid) return;
    const int blk = c >> 2;
    const int E = mx_exponent(a);
    const float inv = mx_inv_scale(E);
    float g[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) g[e] = __fmul_rn(f[e], inv);
    xq[static_cast<size_t>(m) * nchunk + c] = e2m1x8(g);
    if ((threadIdx.x & 3) == 0) xs_atoms[sf_atom_offset(m, blk, atoms_k)] = static_cast<uint8_t>(E + 127);
    if (c < nchunk_s) {
        // the slice's own block over its first r columns (zeros beyond r)
        const int Es = mx_exponent(as);
        const float invs = mx_inv_scale(Es);
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = (c * 8 + e < r) ? __fmul_rn(f[e], invs) : 0.0f;
        xsq[static_cast<size_t>(m) * nchunk_s + c] = e2m1x8(g);
        if ((threadIdx.x & 3) == 0) xss_atoms[sf_atom_offset(m, blk, atoms_s)] = static_cast<uint8_t>(Es + 127);
    }
}

// MXFP4, one CTA per row; four consecutive threads share one 32-element block.
template <class Src>
__device__ __forceinline__ void quant_row_mxfp4(const Src& src, int m, int K, int r, int rp,
                                                uint32_t* __restrict__ xq, uint8_t* __restrict__ xs_atoms,
                                                uint32_t* __restrict__ xsq, uint8_t* __restrict__ xss_atoms) {
    const int nchunk = K >> 3;
    const int atoms_k = (K / 32 + 3) / 4;
    const int atoms_s = (rp / 32 + 3) / 4;
    const int iters = (nchunk + kQuantThreads - 1) / kQuantThreads;
    for (int j = 0; j < iters; ++j) {
        const int c = threadIdx.x + j * kQuantThreads;
        const bool valid = c < nchunk;
        float f[8];
        if (valid) {
            bf16x8_to_f32(src.chunk(c), f);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = 0.0f;
        }
        mx_chunk_out(f, valid, c, m, r, rp, nchunk, xq, xs_atoms, xsq, xss_atoms, atoms_k, atoms_s);
    }
}

template <int MAXC>
__global__ void __launch_bounds__(kQuantThreads, MAXC <= 2 ? 8 : 1)
quant_act_int8_kernel(const uint4* __restrict__ X, int K, int r, int rp, uint8_t* __restrict__ xq,
                      float* __restrict__ xs, uint8_t* __restrict__ xsq, float* __restrict__ xss) {
    __shared__ float red[64];
    pdl_launch_dependents();
    const int m = blockIdx.x;
    const SrcBf16Row src{X + static_cast<size_t>(m) * (K >> 3)};
    quant_row_int8<MAXC>(src, m, K, r, rp, xq, xs, xsq, xss, red);
}

// MXFP4 serq_quant_act as a stream over X^: an MX block (32 values, four
// 16-byte chunks) needs nothing beyond its own row segment, so no row-wide
// reduction is needed. Grid (ceil(K/8 / QF_CHUNKS), M): a CTA owns one
// segment of QF_CHUNKS chunks of one row, each warp QF_UNROLL groups of 32
// consecutive chunks (the four chunks of a block in four consecutive lanes),
// all of its loads issued before any is used. The row is blockIdx.y, so the
// addressing is a few adds; the salient slice is handled only by groups that
// reach into the first rp columns.
constexpr int QF_UNROLL = 4;
constexpr int QF_THREADS = 128;
constexpr int QF_CHUNKS = QF_THREADS * QF_UNROLL;  // 512 chunks = 4096 values of a row per CTA

__global__ void __launch_bounds__(QF_THREADS)
quant_act_mxfp4_flat_kernel(const uint4* __restrict__ X, int K, int r, int rp, uint32_t* __restrict__ xq,
                            uint8_t* __restrict__ xs_atoms, uint32_t* __restrict__ xsq,
                            uint8_t* __restrict__ xss_atoms) {
    pdl_launch_dependents();  // a programmatically launched consumer waits for this grid before reading
    const int nchunk = K >> 3;
    const int nchunk_s = rp >> 3;
    const int m = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int c_base = blockIdx.x * QF_CHUNKS + (threadIdx.x >> 5) * (32 * QF_UNROLL);
    const uint4* row = X + static_cast<size_t>(m) * nchunk;
    uint4 v[QF_UNROLL];
#pragma unroll
    for (int u = 0; u < QF_UNROLL; ++u) {
        const int cc = c_base + u * 32 + lane;
        v[u] = cc < nchunk ? __ldcs(row + cc) : make_uint4(0u, 0u, 0u, 0u);
    }
    // this row's scale atoms: row part of the offset fixed, block part per lane
    const int atoms_k = (K / 32 + 3) / 4;
    const int atoms_s = (rp / 32 + 3) / 4;
    const size_t row_sf = static_cast<size_t>(m & 31) * 16 + static_cast<size_t>((m >> 5) & 3) * 4;
    uint8_t* xs_row = xs_atoms + static_cast<size_t>(m >> 7) * atoms_k * 512 + row_sf;
    uint32_t* xq_row = xq + static_cast<size_t>(m) * nchunk;
#pragma unroll
    for (int u = 0; u < QF_UNROLL; ++u) {
        const int g0 = c_base + u * 32;
        if (g0 >= nchunk) break;                       // warp-uniform
        const int cc = g0 + lane;
        const bool valid = cc < nchunk;                // uniform over each block of four lanes
        float f[8];
        bf16x8_to_f32(v[u], f);
        float a = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(f[e]));
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
        // the salient slice: its own block maximum over the first r columns
        const bool slice_group = g0 < nchunk_s;       // warp-uniform (nchunk_s is a multiple of 8)
        float as = 0.0f;
        if (slice_group) {
            if (valid && cc < nchunk_s) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (cc * 8 + e < r) as = fmaxf(as, fabsf(f[e]));
            }
            as = fmaxf(as, __shfl_xor_sync(0xFFFFFFFFu, as, 1));
            as = fmaxf(as, __shfl_xor_sync(0xFFFFFFFFu, as, 2));
        }
        if (!valid) continue;
        const int blk = cc >> 2;
        const int E = mx_exponent(a);
        const float inv = mx_inv_scale(E);
        float g[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = __fmul_rn(f[e], inv);
        xq_row[cc] = e2m1x8(g);
        if ((lane & 3) == 0) xs_row[(blk >> 2) * 512 + (blk & 3)] = static_cast<uint8_t>(E + 127);
        if (slice_group && cc < nchunk_s) {
            const int Es = mx_exponent(as);
            const float invs = mx_inv_scale(Es);
#pragma unroll
            for (int e = 0; e < 8; ++e) g[e] = (cc * 8 + e < r) ? __fmul_rn(f[e], invs) : 0.0f;
            xsq[static_cast<size_t>(m) * nchunk_s + cc] = e2m1x8(g);
            if ((lane & 3) == 0)
                xss_atoms[static_cast<size_t>(m >> 7) * atoms_s * 512 + row_sf + (blk >> 2) * 512 + (blk & 3)] =
                    static_cast<uint8_t>(Es + 127);
        }
    }
}

// serq_quant_act: one CTA per token row of X^ (bf16, row-major).
template <int MAXC>
__global__ void __launch_bounds__(kQuantThreads, MAXC <= 2 ? 8 : 1)
quant_act_int4_kernel(const uint4* __restrict__ X, int K, int r, int rp, uint32_t* __restrict__ xq,
                      float* __restrict__ xs, uint32_t* __restrict__ xsq, float* __restrict__ xss) {
    __shared__ float red[64];
    pdl_launch_dependents();  // a programmatically launched consumer waits for this grid before reading
    const int m = blockIdx.x;
    const SrcBf16Row src{X + static_cast<size_t>(m) * (K >> 3)};
    quant_row_int4<MAXC>(src, m, K, r, rp, xq, xs, xsq, xss, red);
}


}  // namespace serq
