// serq_linear, MXFP4: Y = bf16( X^_q W^_q^T + X~_{s,q} Q(R)^T ) in one launch.
//
// "量化推理" (reading notes, Stage 2): the residual product needs no
// intermediate quantization, so it is run as ceil(rp / 256) extra K-tiles of
// the same tcgen05 pipeline; both products carry their own E8M0 block scales
// and accumulate into the same fp32 tile in tensor memory.
//
// Tile: 128 tokens x 256 output channels; K-tile: 256 E2M1 elements (128 B).
// Warp roles (persistent, one CTA per SM):
//   warp 0      : TMA producer (codes by tensor-map tile loads, scale atoms by
//                 bulk copies) into a STAGES-deep shared-memory ring
//   warp 1      : owns tensor memory; one lane issues tcgen05.cp (scales) and
//                 tcgen05.mma (kind::mxf4.block_scale, K = 64 per instruction)
//   warps 2..9  : epilogue; each warp drains 32 rows x 128 columns of the
//                 accumulator with tcgen05.ld, releases it, converts to bf16
//                 and stores.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace serq {
namespace mx {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;                 // 256 E2M1 codes per row per K-tile
constexpr int BK = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;        // 16 KB
constexpr int B_BYTES = BN * BK_BYTES;        // 32 KB
constexpr int SFA_BYTES = 2 * 512;            // 128 rows x 8 scales (2 atoms)
constexpr int SFB_BYTES = 4 * 512;            // 256 rows x 8 scales (2 row halves x 2 atoms)
constexpr int NUM_EPI_WARPS = 8;
constexpr int THREADS = 64 + NUM_EPI_WARPS * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_ACC = 0;              // 256 fp32 columns
constexpr uint32_t TMEM_SFA = 256;            // 2 atoms x 4 columns
constexpr uint32_t TMEM_SFB = 264;            // 2 atoms x 8 columns
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) + 1024 /*align*/ + 256 /*barriers*/;

}  // namespace mx

struct MxParams {
    int M, N, K, rp;
    int num_m_tiles, num_tiles;
    int k_tiles_main, k_tiles_res;
    int atoms_k_main;  // K / 128
    int atoms_k_res;   // ceil(rp / 128)
    const uint8_t* sfa;    // activation scale atoms (main)
    const uint8_t* sfb;    // weight scale atoms (main)
    const uint8_t* sfa_r;  // salient-slice scale atoms
    const uint8_t* sfb_r;  // residual scale atoms
    __nv_bfloat16* Y;
};

__global__ void __launch_bounds__(mx::THREADS, 1)
serq_linear_mxfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_ar, const __grid_constant__ CUtensorMap tm_br,
                         const MxParams p) {
    using namespace mx;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * A_BYTES;
    uint8_t* sSFA = sB + STAGES * B_BYTES;
    uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * SFB_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
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
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                const int m_blk = tile % p.num_m_tiles;
                const int n_blk = tile / p.num_m_tiles;
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, 0x101u)) {
                        ok = false;
                        break;
                    }
                    const bool res = kt >= p.k_tiles_main;
                    const int kk = res ? kt - p.k_tiles_main : kt;
                    const int atoms = res ? p.atoms_k_res : p.atoms_k_main;
                    const int na = min(2, atoms - 2 * kk);
                    const uint8_t* sfa_src = res ? p.sfa_r : p.sfa;
                    const uint8_t* sfb_src = res ? p.sfb_r : p.sfb;
                    const bool hi_half = (n_blk * BN + 128) < p.N;
                    const uint32_t sf_bytes = static_cast<uint32_t>(na * 512) * (hi_half ? 3u : 2u);
                    mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES + sf_bytes);
                    tma_load_2d(sA + s * A_BYTES, res ? &tm_ar : &tm_a, &full[s], kk * BK_BYTES, m_blk * BM);
                    tma_load_2d(sB + s * B_BYTES, res ? &tm_br : &tm_b, &full[s], kk * BK_BYTES, n_blk * BN);
                    bulk_load(sSFA + s * SFA_BYTES,
                              sfa_src + (static_cast<size_t>(m_blk) * atoms + 2 * kk) * 512, na * 512, &full[s]);
                    bulk_load(sSFB + s * SFB_BYTES,
                              sfb_src + (static_cast<size_t>(2 * n_blk) * atoms + 2 * kk) * 512, na * 512, &full[s]);
                    if (hi_half)
                        bulk_load(sSFB + s * SFB_BYTES + 1024,
                                  sfb_src + (static_cast<size_t>(2 * n_blk + 1) * atoms + 2 * kk) * 512, na * 512,
                                  &full[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // wait until the MMAs have released every stage before exiting
            for (int i = 0; i < STAGES && ok; ++i) {
                ok = mbar_wait(&empty[s], ph ^ 1u, 0x102u);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, acc_ph = 0;
            bool ok = true;
            const uint32_t idesc_even = idesc_mxf4(BM, BN, 0, 0);
            const uint32_t idesc_odd = idesc_mxf4(BM, BN, 2, 2);
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(acc_empty, acc_ph ^ 1u, 0x201u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&full[s], ph, 0x202u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const bool res = kt >= p.k_tiles_main;
                    const int kk = res ? kt - p.k_tiles_main : kt;
                    const int width = res ? p.rp : p.K;
                    const int steps = min(4, (width - kk * BK) / 64);
                    const int na = (steps + 1) / 2;
                    const uint32_t a_base = smem_u32(sA + s * A_BYTES);
                    const uint32_t b_base = smem_u32(sB + s * B_BYTES);
                    const uint32_t sfa_base = smem_u32(sSFA + s * SFA_BYTES);
                    const uint32_t sfb_base = smem_u32(sSFB + s * SFB_BYTES);
                    for (int j = 0; j < na; ++j) {
                        tc_cp_32x128b_warpx4(tmem + TMEM_SFA + 4 * j, sdesc_sf_atom(sfa_base + 512 * j));
                        tc_cp_32x128b_warpx4(tmem + TMEM_SFB + 8 * j, sdesc_sf_atom(sfb_base + 512 * j));
                        tc_cp_32x128b_warpx4(tmem + TMEM_SFB + 8 * j + 4, sdesc_sf_atom(sfb_base + 1024 + 512 * j));
                    }
                    for (int st = 0; st < steps; ++st) {
                        tc_mma_mxf4(tmem + TMEM_ACC, sdesc_kmajor_sw128(a_base + 32 * st),
                                    sdesc_kmajor_sw128(b_base + 32 * st), (st & 1) ? idesc_odd : idesc_even,
                                    tmem + TMEM_SFA + 4 * (st >> 1), tmem + TMEM_SFB + 8 * (st >> 1),
                                    (kt > 0 || st > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(acc_full);
                acc_ph ^= 1u;
            }
            // drain: all issued tensor-core work has finished before TMEM is freed
            tc_commit(drain);
            mbar_wait(drain, 0, 0x203u);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;             // 0..7
        const int quad = warp & 3;           // TMEM lane quadrant this warp may access
        const int half = ew >> 2;            // columns [128*half, 128*half + 128)
        uint32_t acc_ph = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            const int m_blk = tile % p.num_m_tiles;
            const int n_blk = tile / p.num_m_tiles;
            // warp-uniform wait: the tcgen05.ld below is .sync.aligned
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, acc_ph, 0x301u))) break;
            acc_ph ^= 1u;
            tc_fence_after();
            const uint32_t t_row = tmem + (static_cast<uint32_t>(quad * 32) << 16) + TMEM_ACC + 128u * half;
            uint32_t packed[64];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_row + 32u * c, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    packed[c * 16 + i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            }
            tc_fence_before();
            mbar_arrive(acc_empty);
            const int row = m_blk * BM + quad * 32 + lane;
            const int col0 = n_blk * BN + 128 * half;
            if (row < p.M && col0 < p.N) {
                uint4* out = reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(row) * p.N + col0);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    out[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace serq
