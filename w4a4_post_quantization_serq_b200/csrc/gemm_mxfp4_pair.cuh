// serq_linear, MXFP4, prefill on a CTA pair (cluster of 2, tcgen05 cta_group::2).
//
// Same product as serq_linear_mxfp4_kernel ("量化推理": main K-tiles, then the
// residual's K-tiles, one fp32 accumulator), on a 256 x 256 output tile per
// CTA pair. Each CTA loads its own 128 rows of A and its own 128-row half of
// B; one thread of the even CTA issues M = 256 MMAs that read both CTAs'
// shared memory and write each CTA's 128 rows of D into that CTA's tensor
// memory. Per CTA a K-tile stage holds half the weight rows of the single-CTA
// 128 x 256 tile (41 KB with the wide weight scales, 5 stages).
//
// Warp roles (each CTA): 0 TMA producer; 1 TMEM owner (+ MMA issuer in the
// even CTA); 2 idle; 3..10 epilogue (tcgen05.ld -> release -> bf16 -> store).
//
// Loads: codes and scale atoms all arrive by TMA tile loads. Both CTAs' loads
// of a stage count their bytes on the even CTA's "full" barrier
// (.cta_group::2), which the even CTA's producer arms with the bytes of both;
// the MMA issuer waits on that one barrier, so a stage is handed over in a
// single hop.
//
// Scale atoms reach tensor memory by tcgen05.cp, which the tensor pipe runs
// in order with the MMAs: each copy costs pipe time between K-tiles, so every
// scale tile is copied in the "wide" form one .128x256b copy moves (each
// 512 B atom repeated four times so that every 32-lane quarter of tensor
// memory gets its rows, two atoms side by side): 3 copies per K-tile instead
// of 6 narrow .32x128b.warpx4 ones. The weight scales are stored wide at
// prepare (each 4 KB piece: one K-atom, both 128-row halves of the pair
// tile). The activation scales arrive per call in the canonical atom layout;
// four 3-D TMA loads of the K-tile's two atoms (1 KB, served from L2 after the
// first) build their 4 KB wide tile in shared memory.
//
// Epilogue stores: a thread holds one output row, so storing straight from
// registers would make every warp store touch 32 rows with 16 B each (half
// sectors, 32 L2 requests per instruction). Instead the two warps of a lane
// quadrant take turns passing 64-column slices through a shared 4 KB tile
// (swizzled, conflict-free) and store them eight threads per row: four full
// 128 B lines per instruction.
//
// Two accumulators alternate between tiles so the epilogue of one tile
// overlaps the MMAs of the next. Two 256-column fp32 tiles and the scale
// factors do not fit the 512 tensor-memory columns, so the buffers overlap in
// 24 columns: [0, 256) and [232, 488), scales in [488, 512). The epilogue
// drains the shared columns [232, 256) first and signals "overlap free"; the
// next tile's MMAs wait only for that signal (and for their own buffer's
// previous tile to be fully drained).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_mxfp4.cuh"

namespace serq {
namespace mxp {

constexpr int BM = 128;                       // rows of A per CTA (pair tile: 256)
constexpr int BN = 256;                       // output channels per pair tile
constexpr int BN_HALF = 128;                  // rows of B per CTA
constexpr int BK_BYTES = 128;
constexpr int BK = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;        // 16 KB
constexpr int B_BYTES = BN_HALF * BK_BYTES;   // 16 KB
constexpr int SFA_BYTES = 4 * 2 * 512;        // own 128 rows x 8 scales, wide (4 replicas of 2 atoms)
constexpr int SFB_BYTES = 2 * 4096;           // all 256 rows x 8 scales, wide layout (2 atom pairs)
constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // bytes one CTA loads per stage
constexpr int NUM_EPI_WARPS = 8;
constexpr int EPI_WARP0 = 3;
constexpr int THREADS = (EPI_WARP0 + NUM_EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_ACC0 = 0;
constexpr uint32_t TMEM_ACC1 = 232;           // shares columns [232, 256) with buffer 0
constexpr uint32_t OVL_LO = 232;              // first shared column
constexpr uint32_t TMEM_SFA = 488;
constexpr uint32_t TMEM_SFB = 496;
constexpr int STAGE_OUT_BYTES = 32 * 128;     // per lane quadrant: 32 rows x 64 bf16
// the dynamic shared memory is declared 1024-byte aligned (128 B swizzle), so no pad
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) + 4 * STAGE_OUT_BYTES + 256;

}  // namespace mxp

struct MxPairParams {
    int M, N, K, rp;
    int num_n_tiles, num_tiles;     // pair tiles, m fastest: the CTA pairs working at one time
    int num_m_pairs;                // share weight tiles in L2 (tile = n_blk * num_m_pairs + m_pair)
    int k_tiles_main, k_tiles_res;
    int atoms_k_main, atoms_k_res;
    __nv_bfloat16* Y;
    // SwiGLU epilogue (EPI = 1): tile n_blk's columns are the gate (first 128) and
    // up (last 128) outputs of the down linear's permuted input positions
    // [128 n_blk, +128); the epilogue writes down's quantized input instead of Y.
    int F, r_d, rp_d;               // down's K, rank and padded rank
    const float* inv_s_d;           // [F] 1 / s_down[perm_down[i]]
    uint32_t* hq;                   // [M][F / 8] words of eight E2M1 codes
    uint8_t* hs;                    // E8M0 atoms over (M rows, F / 32 blocks)
    uint32_t* hsq;                  // [M][rp_d / 8] salient slice codes
    uint8_t* hss;                   // E8M0 atoms over (M rows, rp_d / 32 blocks)
    __nv_bfloat16* xhat;            // NULL, or [M][F] debug copy of down's X^
};

// SwiGLU epilogue of one 32-channel block of one row: X^ = bf16(silu(g) u / s)
// for permuted channels i0 .. i0+31, then the MX block (and, inside the first
// r_d channels, the salient slice's own block) written as down's input.
__device__ __forceinline__ void swiglu_quant_block(const MxPairParams& p, int m, int i0, const uint32_t (&g)[32],
                                                   const uint32_t (&u)[32]) {
    float x[32];
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const float gv = __uint_as_float(g[e]);
        const float uv = __uint_as_float(u[e]);
        // fast exp and division: the result is rounded to bf16 (8 bits) right after
        const float silu = __fdividef(gv, 1.0f + __expf(-gv));
        const float v = __fmul_rn(__fmul_rn(silu, uv), __ldg(p.inv_s_d + i0 + e));
        x[e] = __bfloat162float(__float2bfloat16_rn(v));  // the bf16 X^ a stored producer output holds
        amax = fmaxf(amax, fabsf(x[e]));
    }
    const int atoms_f = (p.F / 32 + 3) / 4;
    const int E = mx_exponent(amax);
    const float inv = mx_inv_scale(E);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = __fmul_rn(x[8 * q + e], inv);
        w[q] = e2m1x8(t);
    }
    const size_t row_words = static_cast<size_t>(p.F) / 8;
    *reinterpret_cast<uint4*>(p.hq + static_cast<size_t>(m) * row_words + i0 / 8) = make_uint4(w[0], w[1], w[2], w[3]);
    p.hs[sf_atom_offset(m, i0 / 32, atoms_f)] = static_cast<uint8_t>(E + 127);
    if (i0 < p.rp_d) {
        // the slice's own block: the same block when it lies inside [0, r_d), else
        // its absmax over the channels below r_d (zeros past r_d)
        uint32_t ws[4] = {w[0], w[1], w[2], w[3]};
        int Es = E;
        if (i0 + 32 > p.r_d) {
            float as = 0.0f;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (i0 + e < p.r_d) as = fmaxf(as, fabsf(x[e]));
            Es = mx_exponent(as);
            const float invs = mx_inv_scale(Es);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float t[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = (i0 + 8 * q + e < p.r_d) ? __fmul_rn(x[8 * q + e], invs) : 0.0f;
                ws[q] = e2m1x8(t);
            }
        }
        *reinterpret_cast<uint4*>(p.hsq + static_cast<size_t>(m) * (p.rp_d / 8) + i0 / 8) =
            make_uint4(ws[0], ws[1], ws[2], ws[3]);
        p.hss[sf_atom_offset(m, i0 / 32, (p.rp_d / 32 + 3) / 4)] = static_cast<uint8_t>(Es + 127);
    }
    if (p.xhat != nullptr) {
        uint4* d = reinterpret_cast<uint4*>(p.xhat + static_cast<size_t>(m) * p.F + i0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            d[q] = make_uint4(pack_bf16x2(x[8 * q], x[8 * q + 1]), pack_bf16x2(x[8 * q + 2], x[8 * q + 3]),
                              pack_bf16x2(x[8 * q + 4], x[8 * q + 5]), pack_bf16x2(x[8 * q + 6], x[8 * q + 7]));
    }
}

// Scale tensor maps (reads past the end give zeros). Activation atoms as a
// 3-D view (x: 128 bytes, atom: stride 512, piece: stride 128) with box
// 128 x 2 x 4: one load gives both atoms of a K-tile as 32 row groups of 128 B
// in wide order (piece-major, then atom); wide weight scales as rows of 256 B
// with box 256 x 32 (two 4 KB pieces).
struct MxPairScaleMaps {
    CUtensorMap sfa, sfb, sfa_r, sfb_r;
};

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mxp::THREADS, 1)
serq_linear_mxfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                              const __grid_constant__ CUtensorMap tm_ar, const __grid_constant__ CUtensorMap tm_br,
                              const __grid_constant__ MxPairScaleMaps sf, const MxPairParams p) {
    using namespace mxp;
    extern __shared__ __align__(1024) uint8_t smem_pair[];
    uint8_t* smem = smem_pair;
    if ((smem_u32(smem) & 1023u) != 0) {  // same in both CTAs of the pair: neither reaches a cluster barrier
        if (threadIdx.x == 0) record_timeout(0x1A1u);
        return;
    }
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * A_BYTES;
    uint8_t* sSFA = sB + STAGES * B_BYTES;
    uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
    uint8_t* sOut = sSFB + STAGES * SFB_BYTES;                                // epilogue store tiles
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + 4 * STAGE_OUT_BYTES);  // even CTA: both CTAs' loads landed
    uint64_t* empty = full + STAGES;      // stage consumed (multicast commit)
    uint64_t* acc_full = empty + STAGES;  // [2] accumulator complete (multicast commit)
    uint64_t* acc_empty = acc_full + 2;   // [2] even CTA: both epilogues drained the accumulator
    uint64_t* ovl_empty = acc_empty + 2;  // even CTA: both epilogues drained the shared columns
    uint64_t* drain = ovl_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const int num_clusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * NUM_EPI_WARPS * 32);
        }
        mbar_init(ovl_empty, 2 * 4 * 32);  // the four warps that own the shared columns, both CTAs
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&sf.sfa);
        tma_prefetch_desc(&sf.sfb);
        if (p.k_tiles_res > 0) {
            tma_prefetch_desc(&tm_ar);
            tma_prefetch_desc(&tm_br);
            tma_prefetch_desc(&sf.sfa_r);
            tma_prefetch_desc(&sf.sfb_r);
        }
    }
    cluster_sync();
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM of both allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int total_k = p.k_tiles_main + p.k_tiles_res;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);  // the even CTA's barriers
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = cluster; tile < p.num_tiles && ok; tile += num_clusters) {
                const int n_blk = tile / p.num_m_pairs;
                const int m_pair = tile % p.num_m_pairs;
                const int a_rowblk = 2 * m_pair + static_cast<int>(rank);
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, 0x131u)) {
                        ok = false;
                        break;
                    }
                    const bool res = kt >= p.k_tiles_main;
                    const int kk = res ? kt - p.k_tiles_main : kt;
                    const int atoms = res ? p.atoms_k_res : p.atoms_k_main;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2u * STAGE_TX);
                    const uint32_t bar = full0 + 8u * static_cast<uint32_t>(s);
                    tma_load_2d_pair(sA + s * A_BYTES, res ? &tm_ar : &tm_a, bar, kk * BK_BYTES, a_rowblk * BM);
                    tma_load_2d_pair(sB + s * B_BYTES, res ? &tm_br : &tm_b, bar, kk * BK_BYTES,
                                     n_blk * BN + static_cast<int>(rank) * BN_HALF);
                    // activation scale atoms (2 per K-tile), four replicas = the wide tile
#pragma unroll
                    for (int rep = 0; rep < 4; ++rep)
                        tma_load_3d_pair(sSFA + s * SFA_BYTES + rep * 1024, res ? &sf.sfa_r : &sf.sfa, bar, 0,
                                         a_rowblk * atoms + 2 * kk, 0);
                    tma_load_2d_pair(sSFB + s * SFB_BYTES, res ? &sf.sfb_r : &sf.sfb, bar, 0,
                                     (n_blk * atoms + 2 * kk) * 16);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            for (int i = 0; i < STAGES && ok; ++i) {
                ok = mbar_wait(&empty[s], ph ^ 1u, 0x132u);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (leader && lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            const uint32_t id_even = idesc_mxf4(2 * BM, BN, 0, 0);
            const uint32_t id_odd = idesc_mxf4(2 * BM, BN, 2, 2);
            int it = 0;  // tiles issued by this pair so far
            for (int tile = cluster; tile < p.num_tiles && ok; tile += num_clusters, ++it) {
                const int b = it & 1;
                // this buffer's previous tile fully drained, and the shared columns of the previous tile
                if (!mbar_wait_cluster(&acc_empty[b], static_cast<uint32_t>(((it >> 1) & 1) ^ 1), 0x231u) ||
                    (it > 0 && !mbar_wait_cluster(ovl_empty, static_cast<uint32_t>((it - 1) & 1), 0x234u))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc_col = b ? TMEM_ACC1 : TMEM_ACC0;
                for (int kt = 0; kt < total_k; ++kt) {
                    if (!mbar_wait_cluster(&full[s], ph, 0x232u)) {
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
                    tc_cp_128x256b_pair(tmem + TMEM_SFA, sdesc_sf_wide(sfa_base));
                    for (int j = 0; j < na; ++j) tc_cp_128x256b_pair(tmem + TMEM_SFB + 8 * j, sdesc_sf_wide(sfb_base + 4096 * j));
                    for (int st = 0; st < steps; ++st) {
                        tc_mma_mxf4_pair(tmem + acc_col, sdesc_kmajor_sw128(a_base + 32 * st),
                                         sdesc_kmajor_sw128(b_base + 32 * st), (st & 1) ? id_odd : id_even,
                                         tmem + TMEM_SFA + 4 * (st >> 1), tmem + TMEM_SFB + 8 * (st >> 1),
                                         (kt > 0 || st > 0) ? 1u : 0u);
                    }
                    tc_commit_pair_mc(&empty[s], 0x3);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair_mc(&acc_full[b], 0x3);
            }
            // drain: every pair MMA has finished before tensor memory is freed
            tc_commit_pair_mc(drain, 0x1);
            mbar_wait(drain, 0, 0x233u);
        }
    } else if (warp >= EPI_WARP0) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - EPI_WARP0;
        const int quad = warp & 3;
        const int half = ew >> 2;
        // the two warps of a lane quadrant (half 0 and half 1) share one 4 KB tile
        const uint32_t out_tile = smem_u32(sOut + quad * STAGE_OUT_BYTES);
        const uint32_t sw = static_cast<uint32_t>(lane) & 7u;
        int it = 0;
        for (int tile = cluster; tile < p.num_tiles; tile += num_clusters, ++it) {
            const int n_blk = tile / p.num_m_pairs;
            const int m_pair = tile % p.num_m_pairs;
            const int b = it & 1;
            // on a timeout the warp skips the tile's work but keeps the tile-share barriers in step
            const bool ok =
                __all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[b], static_cast<uint32_t>((it >> 1) & 1), 0x331u));
            if constexpr (EPI == 1) {
                // SwiGLU epilogue: warp (quad, half) owns rows quad*32.. of this CTA and the
                // permuted down channels [64 half, +64) of the tile: two 32-channel blocks,
                // each read as its gate and up columns. The block holding the columns both
                // accumulators share goes first (buffer 0: half 1, block 1 = up columns
                // 224..255; buffer 1: half 0, block 0 = gate columns 0..31).
                if (ok) {
                    tc_fence_after();
                    const uint32_t base = b ? TMEM_ACC1 : TMEM_ACC0;
                    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16) + base;
                    const int m = m_pair * 2 * BM + static_cast<int>(rank) * BM + quad * 32 + lane;
                    const bool owns_ovl = (b == 0 && half == 1) || (b == 1 && half == 0);
                    const int first = b == 0 ? 1 : 0;
#pragma unroll 1
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = owns_ovl ? (jj == 0 ? first : 1 - first) : jj;
                        const int ch0 = 64 * half + 32 * j;
                        uint32_t g[32], u[32];
                        tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(ch0), g);
                        tmem_ld_32x32b_x32(t_lane + 128u + static_cast<uint32_t>(ch0), u);
                        tmem_ld_wait();
                        if (owns_ovl && jj == 0) {
                            tc_fence_before();
                            mbar_arrive_cluster(ovl_empty, 0);
                        }
                        if (m < p.M) swiglu_quant_block(p, m, n_blk * 128 + ch0, g, u);
                    }
                    tc_fence_before();
                    mbar_arrive_cluster(&acc_empty[b], 0);
                }
                continue;
            }
            uint32_t packed[64];
            if (ok) {
                tc_fence_after();
                const uint32_t base = b ? TMEM_ACC1 : TMEM_ACC0;
                const uint32_t t_row = tmem + (static_cast<uint32_t>(quad * 32) << 16) + base + 128u * half;
                // the 32-column chunk of this warp holding the shared columns [232, 256), or -1
                const int c_ovl = (b == 0 && half == 1) ? 3 : ((b == 1 && half == 0) ? 0 : -1);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (c == c_ovl) {  // warp-uniform
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(t_row + 32u * c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            packed[c * 16 + i] =
                                pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                        tc_fence_before();
                        mbar_arrive_cluster(ovl_empty, 0);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (c == c_ovl) continue;
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_row + 32u * c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        packed[c * 16 + i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                }
                tc_fence_before();
                mbar_arrive_cluster(&acc_empty[b], 0);
            }
            const int row0 = m_pair * 2 * BM + static_cast<int>(rank) * BM + quad * 32;  // this warp's rows
            const int col0 = n_blk * BN + 128 * half;
            // four rounds per tile over the shared tile: half 0's two 64-column slices,
            // then half 1's. The owner writes its 32 rows x 128 B (16 B chunk c of row
            // r at slot c ^ (r & 7): conflict-free), then stores them eight threads per
            // row: 4 full 128 B lines per instruction.
#pragma unroll
            for (int round = 0; round < 4; ++round) {
                if (ok && (round >> 1) == half && col0 < p.N) {  // warp-uniform
                    const int cc = (round & 1) * 32;              // first packed word of the slice
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        st_shared_v4(out_tile + static_cast<uint32_t>(lane) * 128u + ((static_cast<uint32_t>(c) ^ sw) << 4),
                                     packed[cc + 4 * c], packed[cc + 4 * c + 1], packed[cc + 4 * c + 2],
                                     packed[cc + 4 * c + 3]);
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = i * 4 + (lane >> 3);
                        const uint32_t slot = static_cast<uint32_t>(lane) & 7u;
                        const uint4 v = ld_shared_v4(out_tile + static_cast<uint32_t>(r) * 128u + (slot << 4));
                        const uint32_t c = slot ^ (static_cast<uint32_t>(r) & 7u);
                        const int grow = row0 + r;
                        if (grow < p.M)
                            *reinterpret_cast<uint4*>(p.Y + static_cast<size_t>(grow) * p.N + col0 + (round & 1) * 64 +
                                                      c * 8) = v;
                    }
                }
                named_bar_sync(1 + quad, 64);  // the shared tile is free for the next round
            }
        }
    }

    tc_fence_before();
    cluster_sync();  // the peer's remote arrivals and the pair MMAs are done
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
}

}  // namespace serq
