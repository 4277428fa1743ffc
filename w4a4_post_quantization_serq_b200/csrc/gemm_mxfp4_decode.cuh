// serq_linear, MXFP4, small M (decode; M <= 16): the same product as the
// prefill kernel, organised to stream W^_q and Q(R) from HBM at full rate.
//
//  * swap-AB: the weight tile (128 output channels) is the MMA's A operand
//    (M_mma = 128) and the <= 16 tokens are its B operand (N_mma = 8 or 16),
//    so no tensor-core rows are spent on padding tokens;
//  * split-K: the K-tiles of the main product followed by the residual's
//    K-tiles ("量化推理": one extra r x N product, no intermediate
//    quantization) are cut into S contiguous ranges; CTA (n_blk, split)
//    streams 128 weight rows over its range;
//  * split reduction, two forms (template flag):
//    - cluster: the S split CTAs of an output block form one thread-block
//      cluster (1 x S x 1). CTA c owns the block's output channels
//      [c R, c R + R) (R = ceil(128 / S) rounded up to 4). Each split sends
//      its fp32 partial sums of the channels a peer owns straight into that
//      peer's shared memory (st.async, 16 bytes at a time, counted on the
//      peer's "received" mbarrier) and stores those it owns itself, so no CTA
//      waits for its peers except for the partial sums it owns: the owner
//      adds the S partials in split order and writes bf16 Y. One cluster
//      barrier, at set-up, makes the peers' mbarriers visible before the
//      first send. No workspace.
//    - workspace: each CTA writes its partial sums to a global workspace; the
//      last CTA of an output block (ticket counter) adds the S partials in
//      split order, writes bf16 Y and resets the counter for the next call.
//    Both add in split order from 0, so results do not depend on scheduling
//    and the two forms agree bit for bit;
//  * programmatic dependent launch: after its set-up each CTA lets the next
//    kernel of the stream start, and the weight tiles of the first stages are
//    requested before waiting for the preceding kernel; token data is read,
//    and the workspace and Y are written, only after that wait. Weight
//    streaming of consecutive linears thus overlaps the previous one's tail.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_mxfp4.cuh"

namespace serq {
namespace mxd {

constexpr int BM = 128;                 // output channels per CTA
constexpr int BK = 256;                 // codes per K-tile
constexpr int BK_BYTES = 128;
constexpr int MAX_TOKENS = 16;
constexpr int STAGES = 5;
constexpr int A_BYTES = BM * BK_BYTES;           // 16 KB weight codes
constexpr int B_BYTES = MAX_TOKENS * BK_BYTES;   // 2 KB token codes
constexpr int SFA_BYTES = 2 * 512;               // weight scale atoms
constexpr int SFB_BYTES = 2 * 512;               // token scale atoms
constexpr int THREADS = 64 + 4 * 32;             // producer, MMA, 4 epilogue warps
constexpr uint32_t TMEM_COLS = 32;
constexpr uint32_t TMEM_ACC = 0;                 // 16 fp32 columns (tokens)
constexpr uint32_t TMEM_SFA = 16;                // 2 atoms x 4 columns
constexpr uint32_t TMEM_SFB = 24;                // 2 atoms x 4 columns
constexpr int MAX_SPLITS = 8;                    // portable cluster size
// partial sums received by an owner (cluster form): [split][owned channel][token],
// at most S * R * 16 * 4 bytes over S <= 8 (S = 6: 6 * 24 * 64 = 9216)
constexpr int PART_BYTES = 9216;
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) + PART_BYTES + 1024 + 256;

}  // namespace mxd

struct MxDecodeParams {
    int M, N, K, rp;
    int n_tokens_mma;       // 8 or 16
    int k_tiles_main, k_tiles_total;
    int splits;
    int atoms_k_main, atoms_k_res;
    const uint8_t* sf_w;    // weight scale atoms (main)
    const uint8_t* sf_x;    // token scale atoms (main)
    const uint8_t* sf_wr;   // residual scale atoms
    const uint8_t* sf_xr;   // salient-slice scale atoms
    float* partial;         // workspace form: [splits][M][N]
    unsigned int* tickets;  // workspace form: [N / 128], zero between calls
    __nv_bfloat16* Y;
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

template <bool kClusterReduce>
__global__ void __launch_bounds__(mxd::THREADS)
serq_linear_mxfp4_decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                                const __grid_constant__ CUtensorMap tm_wr, const __grid_constant__ CUtensorMap tm_xr,
                                const MxDecodeParams p) {
    using namespace mxd;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * A_BYTES;
    uint8_t* sSFA = sB + STAGES * B_BYTES;
    uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
    float* spart = reinterpret_cast<float*>(sSFB + STAGES * SFB_BYTES);  // [split][rows_per][nt]
    uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * SFB_BYTES + PART_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* drain = acc_full + 1;
    uint64_t* recv_full = drain + 1;  // cluster form: every split's partial sums of the owned channels arrived
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv_full + 1);
    __shared__ unsigned int s_is_last;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_blk = blockIdx.x;
    const int split = blockIdx.y;
    const int kt0 = static_cast<int>((static_cast<long long>(p.k_tiles_total) * split) / p.splits);
    const int kt1 = static_cast<int>((static_cast<long long>(p.k_tiles_total) * (split + 1)) / p.splits);
    // cluster form: the cluster spans the S splits of this block, so the CTA's rank is its split
    const int rows_per = ((BM + p.splits - 1) / p.splits + 3) & ~3;
    const int row0 = split * rows_per;
    const int rows_own = min(BM, row0 + rows_per) - row0;
    const int nt = p.n_tokens_mma;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        if constexpr (kClusterReduce) mbar_init(recv_full, 1);
        fence_mbar_init();
        if constexpr (kClusterReduce)
            mbar_arrive_expect_tx(recv_full, static_cast<uint32_t>((p.splits - 1) * rows_own * nt * 4));
        // the token maps are first used right after the wait on the preceding kernel
        tma_prefetch_desc(&tm_x);
        if (p.k_tiles_total > p.k_tiles_main) tma_prefetch_desc(&tm_xr);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if constexpr (kClusterReduce) cluster_arrive();  // this CTA's "received" barrier is initialised
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // weights (independent of the preceding kernel) of the first stages first
            const int pre = min(STAGES, kt1 - kt0);
            for (int i = 0; i < pre; ++i) {
                const int kt = kt0 + i;
                const bool res = kt >= p.k_tiles_main;
                const int kk = res ? kt - p.k_tiles_main : kt;
                const int atoms = res ? p.atoms_k_res : p.atoms_k_main;
                const int na = min(2, atoms - 2 * kk);
                // token box = n_tokens_mma rows
                mbar_arrive_expect_tx(&full[i], A_BYTES + p.n_tokens_mma * BK_BYTES + 2u * na * 512u);
                tma_load_2d(sA + i * A_BYTES, res ? &tm_wr : &tm_w, &full[i], kk * BK_BYTES, n_blk * BM);
                bulk_load(sSFA + i * SFA_BYTES,
                          (res ? p.sf_wr : p.sf_w) + (static_cast<size_t>(n_blk) * atoms + 2 * kk) * 512, na * 512,
                          &full[i]);
            }
            pdl_wait_prerequisites();
            int s = 0;
            uint32_t ph = 0;
            for (int kt = kt0; kt < kt1; ++kt) {
                const bool res = kt >= p.k_tiles_main;
                const int kk = res ? kt - p.k_tiles_main : kt;
                const int atoms = res ? p.atoms_k_res : p.atoms_k_main;
                const int na = min(2, atoms - 2 * kk);
                if (kt - kt0 >= pre) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, 0x121u)) break;
                    mbar_arrive_expect_tx(&full[s], A_BYTES + p.n_tokens_mma * BK_BYTES + 2u * na * 512u);
                    tma_load_2d(sA + s * A_BYTES, res ? &tm_wr : &tm_w, &full[s], kk * BK_BYTES, n_blk * BM);
                    bulk_load(sSFA + s * SFA_BYTES,
                              (res ? p.sf_wr : p.sf_w) + (static_cast<size_t>(n_blk) * atoms + 2 * kk) * 512,
                              na * 512, &full[s]);
                }
                tma_load_2d(sB + s * B_BYTES, res ? &tm_xr : &tm_x, &full[s], kk * BK_BYTES, 0);
                bulk_load(sSFB + s * SFB_BYTES, (res ? p.sf_xr : p.sf_x) + static_cast<size_t>(2 * kk) * 512,
                          na * 512, &full[s]);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // every stage released (all tensor-core reads and barrier arrivals done)
            for (int i = 0; i < STAGES; ++i) {
                if (!mbar_wait(&empty[s], ph ^ 1u, 0x122u)) break;
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
            uint32_t ph = 0;
            bool ok = true;
            const uint32_t id_even = idesc_mxf4(BM, p.n_tokens_mma, 0, 0);
            const uint32_t id_odd = idesc_mxf4(BM, p.n_tokens_mma, 2, 2);
            bool first = true;
            for (int kt = kt0; kt < kt1; ++kt) {
                if (!mbar_wait(&full[s], ph, 0x221u)) {
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
                    tc_cp_32x128b_warpx4(tmem + TMEM_SFB + 4 * j, sdesc_sf_atom(sfb_base + 512 * j));
                }
                for (int st = 0; st < steps; ++st) {
                    tc_mma_mxf4(tmem + TMEM_ACC, sdesc_kmajor_sw128(a_base + 32 * st),
                                sdesc_kmajor_sw128(b_base + 32 * st), (st & 1) ? id_odd : id_even,
                                tmem + TMEM_SFA + 4 * (st >> 1), tmem + TMEM_SFB + 4 * (st >> 1), first ? 0u : 1u);
                    first = false;
                }
                tc_commit(&empty[s]);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (ok) tc_commit(acc_full);
            tc_commit(drain);
            mbar_wait(drain, 0, 0x222u);
        }
    } else {
        // ------------------------------------------------------------ epilogue: partial sums
        const int quad = warp & 3;
        const int n = n_blk * BM + quad * 32 + lane;
        pdl_wait_prerequisites();  // the preceding kernel is done with the workspace and Y
        uint32_t v[16] = {};
        const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, 0x321u));
        if (got) {
            tc_fence_after();
            tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quad * 32) << 16) + TMEM_ACC, v);
            tmem_ld_wait();
        }
        if constexpr (kClusterReduce) {
            // this channel's partial sums (all nt token columns) go to its owner: a
            // peer's by st.async (even after a timed-out wait, so that the owners'
            // barriers complete), this CTA's own by plain stores
            cluster_wait();
            const int row = quad * 32 + lane;
            const int owner = row / rows_per;
            const int slot = ((split * rows_per + row - owner * rows_per) * nt) * 4;  // bytes into spart
            if (owner == split) {
                float4* d = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(spart) + slot);
#pragma unroll
                for (int j = 0; j < MAX_TOKENS / 4; ++j)
                    if (4 * j < nt)
                        d[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                           __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
            } else {
                const uint32_t dst = mapa_shared(smem_u32(spart) + static_cast<uint32_t>(slot),
                                                 static_cast<uint32_t>(owner));
                const uint32_t bar = mapa_shared(smem_u32(recv_full), static_cast<uint32_t>(owner));
#pragma unroll
                for (int j = 0; j < MAX_TOKENS / 4; ++j)
                    if (4 * j < nt)
                        st_async_v4f32(dst + 16u * j, __uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                       __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]), bar);
            }
        } else if (got) {
            float* part = p.partial + static_cast<size_t>(split) * p.M * p.N;
#pragma unroll
            for (int m = 0; m < MAX_TOKENS; ++m)
                if (m < p.M) part[static_cast<size_t>(m) * p.N + n] = __uint_as_float(v[m]);
        }
        tc_fence_before();
    }

    // ---------------------------------------------------------------- split reduction
    pdl_wait_prerequisites();
    if constexpr (kClusterReduce) {
        if (warp < 2) {
            __syncwarp();
            cluster_wait();  // the epilogue warps waited before their sends
        }
        __syncthreads();  // this CTA's own partial sums are in shared memory
        // then the peers' (counted on recv_full); no peer writes this CTA's shared
        // memory after that, so it may leave once it has added them
        if (mbar_wait_cluster(recv_full, 0, 0x323u)) {
            const int groups = p.M * (rows_own / 4);  // (token, 4 consecutive owned channels)
            for (int g = threadIdx.x; g < groups; g += blockDim.x) {
                const int m = g % p.M;
                const int c = 4 * (g / p.M);
                float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                for (int sp = 0; sp < p.splits; ++sp) {
                    const float* src = spart + (sp * rows_per + c) * nt + m;
                    acc.x += src[0];
                    acc.y += src[nt];
                    acc.z += src[2 * nt];
                    acc.w += src[3 * nt];
                }
                uint2 out;
                out.x = pack_bf16x2(acc.x, acc.y);
                out.y = pack_bf16x2(acc.z, acc.w);
                *reinterpret_cast<uint2*>(p.Y + static_cast<size_t>(m) * p.N + n_blk * BM + row0 + c) = out;
            }
        }
    } else {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            const unsigned int ticket = atomicAdd(&p.tickets[n_blk], 1u);
            s_is_last = (ticket == static_cast<unsigned int>(p.splits - 1)) ? 1u : 0u;
        }
        __syncthreads();
        if (s_is_last) {
            __threadfence();
            for (int idx = threadIdx.x; idx < p.M * BM; idx += blockDim.x) {
                const int m = idx / BM;
                const int n = n_blk * BM + idx % BM;
                float acc = 0.0f;
                for (int sp = 0; sp < p.splits; ++sp)
                    acc += __ldcg(p.partial + (static_cast<size_t>(sp) * p.M + m) * p.N + n);
                p.Y[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(acc);
            }
            if (threadIdx.x == 0) p.tickets[n_blk] = 0u;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace serq
