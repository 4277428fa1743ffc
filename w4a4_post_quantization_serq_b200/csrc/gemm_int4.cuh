// serq_linear, INT4 weights (W4A4 and W4A8):
//   acc1 = X^_q W^_q^T (int32, exact),  acc2 = X~_{s,q} Q(R)^T (int32, exact)
//   Y    = bf16(acc1 * s_x[m] * s_w[n] + acc2 * s_xs[m] * s_R[n])
// ("量化推理", reading notes). The two products have different scales, so
// they accumulate into two tensor-memory tiles; the residual runs as extra
// K-tiles of the same pipeline, in the same launch.
//
// sm_100 tensor cores have no 4-bit integer kind, so packed nibbles are
// brought in by TMA and a converter warpgroup sign-extends them into the
// 128-byte-swizzled int8 layout that tcgen05.mma kind::i8 reads.
//   W4A4 (A8 = false): activations and weights are both unpacked.
//   W4A8 (A8 = true) : the activations are already int8 ([-127, 127]), so TMA
//                      loads them straight into the swizzled MMA layout (their
//                      own ring of stages); only the weights are unpacked.
//
// Tile 128 x 256, K-tile 128 codes (4 MMAs of K = 32). Warp roles: 0 producer,
// 1 MMA (+TMEM owner), 2..5 epilogue, 6..9 converters. Each converter thread
// issues all of its shared-memory loads of a tile before unpacking them.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_mxfp4.cuh"

namespace serq {
namespace i4 {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;                     // codes per K-tile
constexpr int PK_BYTES = BK / 2;            // packed bytes per row per K-tile
constexpr int NUM_EPI_WARPS = 4;
constexpr int NUM_CVT_WARPS = 4;
constexpr int CVT_THREADS = NUM_CVT_WARPS * 32;
constexpr int THREADS = 64 + (NUM_EPI_WARPS + NUM_CVT_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_ACC1 = 0;
constexpr uint32_t TMEM_ACC2 = 256;

// Shared-memory plan per variant (all operand tiles 1024-byte aligned).
template <bool A8>
struct Plan {
    static constexpr int STG_STAGES = 3;                   // packed staging (TMA)
    static constexpr int OP_STAGES = 3;                    // unpacked int8 operands (converters)
    static constexpr int A_STAGES = A8 ? 4 : 0;            // W4A8: int8 activations straight from TMA
    static constexpr int STG_A = A8 ? 0 : BM * PK_BYTES;   // 8 KB
    static constexpr int STG_B = BN * PK_BYTES;            // 16 KB
    static constexpr int OP_A = A8 ? 0 : BM * BK;          // 16 KB
    static constexpr int OP_B = BN * BK;                   // 32 KB
    static constexpr int RING_A = A8 ? BM * BK : 0;        // 16 KB
    static constexpr int SMEM_BYTES =
        A_STAGES * RING_A + OP_STAGES * (OP_A + OP_B) + STG_STAGES * (STG_A + STG_B) + 1024 + 512;
};

}  // namespace i4

struct I4Params {
    int M, N, K, rp;
    int num_m_tiles, num_tiles;
    int k_tiles_main, k_tiles_res;
    const float* sx;   // [M]
    const float* sxs;  // [M]
    const float* sw;   // [N]
    const float* sR;   // [N]
    __nv_bfloat16* Y;
    int32_t* acc_dbg;  // NULL or [2][M][N]
};

// 8 packed nibbles (element 0 lowest) -> 8 sign-extended int8 in two words.
__device__ __forceinline__ void nibbles_to_s8(uint32_t w, uint32_t& out0, uint32_t& out1) {
    uint32_t lo = w & 0x0F0F0F0Fu;          // elements 0, 2, 4, 6
    uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // elements 1, 3, 5, 7
    lo |= (lo & 0x08080808u) * 0x1Eu;       // sign bit 3 -> 0xF0 in each byte
    hi |= (hi & 0x08080808u) * 0x1Eu;
    out0 = __byte_perm(lo, hi, 0x5140);     // e0 e1 e2 e3
    out1 = __byte_perm(lo, hi, 0x7362);     // e4 e5 e6 e7
}

// Unpack ROWS x 64 packed bytes (row-major) into ROWS x 128 int8 with the
// 128-byte swizzle: 16-byte chunk c of row r goes to chunk c ^ (r & 7).
// Each of the CVT_THREADS threads loads all of its chunks first.
template <int ROWS>
__device__ __forceinline__ void unpack_tile(const uint8_t* stg, uint8_t* op, int tid) {
    constexpr int TASKS = ROWS * 4;
    constexpr int PER = TASKS / i4::CVT_THREADS;
    static_assert(TASKS % i4::CVT_THREADS == 0, "whole chunks per thread");
    uint4 v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = *reinterpret_cast<const uint4*>(stg + (tid + i * i4::CVT_THREADS) * 16);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int t = tid + i * i4::CVT_THREADS;
        const int r = t >> 2, pc = t & 3;
        uint32_t o[8];
        nibbles_to_s8(v[i].x, o[0], o[1]);
        nibbles_to_s8(v[i].y, o[2], o[3]);
        nibbles_to_s8(v[i].z, o[4], o[5]);
        nibbles_to_s8(v[i].w, o[6], o[7]);
        uint8_t* rowp = op + r * 128;
        *reinterpret_cast<uint4*>(rowp + (((2 * pc) ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(rowp + (((2 * pc + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

template <bool A8>
__global__ void __launch_bounds__(i4::THREADS, 1)
serq_linear_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_ar, const __grid_constant__ CUtensorMap tm_br,
                        const I4Params p) {
    using namespace i4;
    using PL = Plan<A8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* rA = smem;                                       // W4A8: int8 activation ring
    uint8_t* oA = rA + PL::A_STAGES * PL::RING_A;             // W4A4: unpacked activations
    uint8_t* oB = oA + PL::OP_STAGES * PL::OP_A;              // unpacked weights
    uint8_t* gA = oB + PL::OP_STAGES * PL::OP_B;              // packed staging
    uint8_t* gB = gA + PL::STG_STAGES * PL::STG_A;
    uint64_t* stg_full = reinterpret_cast<uint64_t*>(gB + PL::STG_STAGES * PL::STG_B);
    uint64_t* stg_empty = stg_full + PL::STG_STAGES;
    uint64_t* op_full = stg_empty + PL::STG_STAGES;
    uint64_t* op_empty = op_full + PL::OP_STAGES;
    uint64_t* a_full = op_empty + PL::OP_STAGES;              // W4A8 ring (A_STAGES entries)
    uint64_t* a_empty = a_full + (A8 ? PL::A_STAGES : 0);
    uint64_t* acc_full = a_empty + (A8 ? PL::A_STAGES : 0);
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < PL::STG_STAGES; ++s) {
            mbar_init(&stg_full[s], 1);
            mbar_init(&stg_empty[s], CVT_THREADS);
        }
        for (int s = 0; s < PL::OP_STAGES; ++s) {
            mbar_init(&op_full[s], CVT_THREADS);
            mbar_init(&op_empty[s], 1);
        }
        for (int s = 0; s < PL::A_STAGES; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, NUM_EPI_WARPS * 32);
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        if (p.k_tiles_res > 0) {
            tma_prefetch_desc(&tm_ar);
            tma_prefetch_desc(&tm_br);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total_k = p.k_tiles_main + p.k_tiles_res;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int s = 0, sa = 0;
            uint32_t ph = 0, pha = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                const int m_blk = tile % p.num_m_tiles;
                const int n_blk = tile / p.num_m_tiles;
                for (int kt = 0; kt < total_k; ++kt) {
                    const bool res = kt >= p.k_tiles_main;
                    const int kk = res ? kt - p.k_tiles_main : kt;
                    if constexpr (A8) {
                        // int8 activations: 128 codes = 128 bytes per row, straight into the MMA layout
                        if (!mbar_wait(&a_empty[sa], pha ^ 1u, 0x114u)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&a_full[sa], PL::RING_A);
                        tma_load_2d(rA + sa * PL::RING_A, res ? &tm_ar : &tm_a, &a_full[sa], kk * BK, m_blk * BM);
                        if (++sa == PL::A_STAGES) {
                            sa = 0;
                            pha ^= 1u;
                        }
                    }
                    if (!mbar_wait(&stg_empty[s], ph ^ 1u, 0x111u)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&stg_full[s], PL::STG_A + PL::STG_B);
                    if constexpr (!A8)
                        tma_load_2d(gA + s * PL::STG_A, res ? &tm_ar : &tm_a, &stg_full[s], kk * PK_BYTES, m_blk * BM);
                    tma_load_2d(gB + s * PL::STG_B, res ? &tm_br : &tm_b, &stg_full[s], kk * PK_BYTES, n_blk * BN);
                    if (++s == PL::STG_STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            for (int i = 0; i < PL::STG_STAGES && ok; ++i) {
                ok = mbar_wait(&stg_empty[s], ph ^ 1u, 0x112u);
                if (++s == PL::STG_STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            for (int i = 0; i < PL::A_STAGES && ok; ++i) {
                ok = mbar_wait(&a_empty[sa], pha ^ 1u, 0x115u);
                if (++sa == PL::A_STAGES) {
                    sa = 0;
                    pha ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0, sa = 0;
            uint32_t ph = 0, pha = 0, acc_ph = 0;
            bool ok = true;
            const uint32_t idesc = idesc_i8(BM, BN);
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(acc_empty, acc_ph ^ 1u, 0x211u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&op_full[s], ph, 0x212u) || (A8 && !mbar_wait(&a_full[sa], pha, 0x214u))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const bool res = kt >= p.k_tiles_main;
                    const int kk = res ? kt - p.k_tiles_main : kt;
                    const int width = res ? p.rp : p.K;
                    const int steps = min(4, (width - kk * BK) / 32);
                    const uint32_t a_base = A8 ? smem_u32(rA + sa * PL::RING_A) : smem_u32(oA + s * PL::OP_A);
                    const uint32_t b_base = smem_u32(oB + s * PL::OP_B);
                    const uint32_t d = tmem + (res ? TMEM_ACC2 : TMEM_ACC1);
                    for (int st = 0; st < steps; ++st) {
                        const bool acc = res ? (kk > 0 || st > 0) : (kt > 0 || st > 0);
                        tc_mma_i8(d, sdesc_kmajor_sw128(a_base + 32 * st), sdesc_kmajor_sw128(b_base + 32 * st),
                                  idesc, acc ? 1u : 0u);
                    }
                    tc_commit(&op_empty[s]);
                    if (++s == PL::OP_STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if constexpr (A8) {
                        tc_commit(&a_empty[sa]);
                        if (++sa == PL::A_STAGES) {
                            sa = 0;
                            pha ^= 1u;
                        }
                    }
                }
                if (!ok) break;
                tc_commit(acc_full);
                acc_ph ^= 1u;
            }
            tc_commit(drain);
            mbar_wait(drain, 0, 0x213u);
        }
    } else if (warp < 2 + NUM_EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;
        uint32_t acc_ph = 0;
        const bool has_res = p.k_tiles_res > 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            const int m_blk = tile % p.num_m_tiles;
            const int n_blk = tile / p.num_m_tiles;
            // warp-uniform wait: the tcgen05.ld below is .sync.aligned
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, acc_ph, 0x311u))) break;
            acc_ph ^= 1u;
            tc_fence_after();
            const int row = m_blk * BM + quad * 32 + lane;
            const bool row_ok = row < p.M;
            const float sx = row_ok ? p.sx[row] : 0.0f;
            const float sxs = (row_ok && has_res) ? p.sxs[row] : 0.0f;
            const uint32_t t_row = tmem + (static_cast<uint32_t>(quad * 32) << 16);
            for (int c = 0; c < BN / 32; ++c) {
                const int col0 = n_blk * BN + 32 * c;
                uint32_t a1[32], a2[32];
                tmem_ld_32x32b_x32(t_row + TMEM_ACC1 + 32u * c, a1);
                if (has_res) tmem_ld_32x32b_x32(t_row + TMEM_ACC2 + 32u * c, a2);
                tmem_ld_wait();
                if (!has_res) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) a2[i] = 0u;
                }
                if (row_ok && col0 < p.N) {
                    uint32_t packed[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float y[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int n = col0 + i + u;
                            const float f1 = static_cast<float>(static_cast<int32_t>(a1[i + u]));
                            const float f2 = static_cast<float>(static_cast<int32_t>(a2[i + u]));
                            const float g1 = __fmul_rn(sx, __ldg(p.sw + n));
                            const float g2 = has_res ? __fmul_rn(sxs, __ldg(p.sR + n)) : 0.0f;
                            y[u] = __fadd_rn(__fmul_rn(f1, g1), __fmul_rn(f2, g2));
                        }
                        packed[i / 2] = pack_bf16x2(y[0], y[1]);
                    }
                    uint4* out = reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(row) * p.N + col0);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        out[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                    if (p.acc_dbg != nullptr) {
                        int4* d1 = reinterpret_cast<int4*>(p.acc_dbg + static_cast<size_t>(row) * p.N + col0);
                        int4* d2 = reinterpret_cast<int4*>(p.acc_dbg + static_cast<size_t>(p.M) * p.N +
                                                           static_cast<size_t>(row) * p.N + col0);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            d1[i] = make_int4(a1[4 * i], a1[4 * i + 1], a1[4 * i + 2], a1[4 * i + 3]);
                            d2[i] = make_int4(a2[4 * i], a2[4 * i + 1], a2[4 * i + 2], a2[4 * i + 3]);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(acc_empty);
        }
    } else {
        // ------------------------------------------------------------ converters
        const int tid = threadIdx.x - (2 + NUM_EPI_WARPS) * 32;
        int s1 = 0, s2 = 0;
        uint32_t ph1 = 0, ph2 = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
            for (int kt = 0; kt < total_k; ++kt) {
                if (!mbar_wait(&stg_full[s1], ph1, 0x411u) || !mbar_wait(&op_empty[s2], ph2 ^ 1u, 0x412u)) {
                    ok = false;
                    break;
                }
                if constexpr (!A8) unpack_tile<BM>(gA + s1 * PL::STG_A, oA + s2 * PL::OP_A, tid);
                unpack_tile<BN>(gB + s1 * PL::STG_B, oB + s2 * PL::OP_B, tid);
                fence_proxy_async_smem();   // generic-proxy writes -> visible to the tensor cores
                mbar_arrive(&op_full[s2]);
                mbar_arrive(&stg_empty[s1]);
                if (++s1 == PL::STG_STAGES) {
                    s1 = 0;
                    ph1 ^= 1u;
                }
                if (++s2 == PL::OP_STAGES) {
                    s2 = 0;
                    ph2 ^= 1u;
                }
            }
        }
        // wait until the MMAs have consumed every converted stage
        for (int i = 0; i < PL::OP_STAGES && ok; ++i) {
            ok = mbar_wait(&op_empty[s2], ph2 ^ 1u, 0x413u);
            if (++s2 == PL::OP_STAGES) {
                s2 = 0;
                ph2 ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace serq
