// Causal grouped-query attention for the prefill block (head_dim 128) on the
// fifth-generation tensor cores: O_h = softmax(Q_h K_g^T / sqrt(d) + causal
// mask) V_g, g = h / (n_q / n_kv), the standard LLaMA definition.
//
// One CTA per (128 queries, head); 128-key tiles in order up to the block's
// last query. Per key tile j:
//   S_j = Q K_j^T       tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M = 128,
//                       N = 128, K = 128, into one of two tensor-memory buffers;
//   softmax             four warps, one query row per thread (its tensor-memory
//                       lane): scale, mask, running max m and sum l in the
//                       exp2 domain, P_j = exp2(S - m) rounded to bf16 into a
//                       shared-memory tile in the MMA's operand layout;
//   O += P_j V_j        M = 128, N = 128, K = 128, accumulated by the tensor
//                       cores into one fp32 tile in tensor memory.
// P_j is taken against a per-row reference maximum m_ref that moves only when
// the row's running maximum exceeds it by more than TAU (log2 units), so P <=
// 2^TAU. When a row's reference moves, its warp rescales that row of O (and
// of the running sum) in tensor memory by exp2(old - new) between O += P_{j-1}
// V_{j-1} and O += P_j V_j; otherwise nothing but S and P pass through the
// softmax warps. At the end O / l is stored as bf16.
// Q and K tiles arrive by TMA with the 128-byte swizzle (K-major operands);
// V enters the second product as its transpose (dims x keys, K-major), which
// serq_attention_prefill writes first. Warp 0 loads, warp 1 issues the MMAs
// (one thread) and owns tensor memory, warps 2..5 do the softmax.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace serq {
namespace atc {

constexpr int D = 128;                  // head dimension
constexpr int BM = 128;                 // queries per CTA: one per tensor-memory lane
constexpr int BN = 128;                 // keys per tile
constexpr int KB = BN / 64;             // 128-byte column blocks of a key row (P, V^T)
constexpr int STAGES = 2;               // K / V^T tile ring
constexpr int Q_BYTES = BM * D * 2;     // 32 KB: two column blocks of [128 queries][128 B]
constexpr int K_BYTES = BN * D * 2;     // 32 KB: two column blocks of [128 keys][128 B]
constexpr int V_BYTES = D * BN * 2;     // 32 KB: KB column blocks of [128 dims][64 keys = 128 B]
constexpr int P_BYTES = BM * BN * 2;    // 32 KB: KB column blocks of [128 queries][64 keys = 128 B]
constexpr int CB_BYTES = 128 * 128;     // one column block of 128 rows
constexpr int THREADS = 6 * 32;         // warp 0 TMA, 1 MMA, 2..5 softmax
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_S = 0;          // + BN b: S buffers (BN fp32 columns each)
constexpr uint32_t TMEM_O = 2 * BN;     // O accumulator (128 fp32 columns)
constexpr float TAU = 8.0f;             // reference-maximum slack (log2 units): P <= 2^8
constexpr int SMEM_BYTES = 1024 + Q_BYTES + STAGES * (K_BYTES + V_BYTES) + 2 * P_BYTES + 256;

}  // namespace atc

// Instruction descriptor of kind::f16 with bf16 operands, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)     // D format: f32
           | (1u << 7)   // A: bf16
           | (1u << 10)  // B: bf16
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 2^x on the special-function unit (ex2.approx.ftz; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait_att() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct AttTcParams {
    int M, n_q, n_kv;
    float scale_log2;  // log2(e) / sqrt(d)
    __nv_bfloat16* o;
    int ldo;
};

// V^T of each key-value group: vt[(g * 128 + d) * M_pad + m] = v[m * ldkv + g * 128 + d],
// zeros for M <= m < M_pad. Tiles of 32 keys x 32 dims through shared memory.
__global__ void transpose_v_kernel(const __nv_bfloat16* __restrict__ v, int ldkv, int M, int M_pad,
                                   __nv_bfloat16* __restrict__ vt) {
    __shared__ __nv_bfloat16 t[32][33];
    const int k0 = blockIdx.x * 32, d0 = blockIdx.y * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int key = k0 + ty + 8 * i;
        t[ty + 8 * i][tx] = key < M ? v[static_cast<size_t>(key) * ldkv + d0 + tx] : __float2bfloat16(0.0f);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int d = d0 + ty + 8 * i;
        if (k0 + tx < M_pad) vt[static_cast<size_t>(d) * M_pad + k0 + tx] = t[tx][ty + 8 * i];
    }
}

// grid (ceil(M / 128), n_q): CTA (qb, h) computes queries [128 qb, +128) of head h;
// blocks taken last-first so the longest (most keys) start first.
__global__ void __launch_bounds__(atc::THREADS, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_vt, const AttTcParams p) {
    using namespace atc;
    extern __shared__ uint8_t smem_atc[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_atc) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + Q_BYTES;
    uint8_t* sV = sK + STAGES * K_BYTES;
    uint8_t* sP = sV + STAGES * V_BYTES;
    uint64_t* q_full = reinterpret_cast<uint64_t*>(sP + 2 * P_BYTES);
    uint64_t* kv_full = q_full + 1;         // [STAGES]
    uint64_t* kv_empty = kv_full + STAGES;  // [STAGES] (MMA commit)
    uint64_t* s_full = kv_empty + STAGES;   // [2] S_j in tensor memory (MMA commit)
    uint64_t* s_empty = s_full + 2;         // [2] the softmax warps have read S_j
    uint64_t* p_full = s_empty + 2;         // [2] P_j in shared memory
    uint64_t* o_done = p_full + 2;          // [2] O += P_j V_j finished, by tile parity (MMA commit)
    uint64_t* drain = o_done + 2;           // every MMA finished (before tensor memory is freed)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);
    const int h = blockIdx.y;
    const int g = h / (p.n_q / p.n_kv);
    const int q0 = qb * BM;
    const int last_key = min(q0 + BM, p.M);          // keys [0, last_key) can be visible
    const int n_tiles = (last_key + BN - 1) / BN;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 4);
            mbar_init(&p_full[b], 4);
            mbar_init(&o_done[b], 1);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_vt);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, Q_BYTES);
            tma_load_2d(sQ, &tm_q, q_full, (h * D) * 2, q0);
            tma_load_2d(sQ + Q_BYTES / 2, &tm_q, q_full, (h * D + 64) * 2, q0);
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % STAGES;
                if (j >= STAGES && !mbar_wait(&kv_empty[s], static_cast<uint32_t>((j / STAGES - 1) & 1), 0x511u))
                    break;
                mbar_arrive_expect_tx(&kv_full[s], K_BYTES + V_BYTES);
                tma_load_2d(sK + s * K_BYTES, &tm_k, &kv_full[s], (g * D) * 2, j * BN);
                tma_load_2d(sK + s * K_BYTES + K_BYTES / 2, &tm_k, &kv_full[s], (g * D + 64) * 2, j * BN);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_2d(sV + s * V_BYTES + kb * CB_BYTES, &tm_vt, &kv_full[s], (j * BN + 64 * kb) * 2, g * D);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(BM, BN);
            const uint32_t id_o = idesc_bf16(BM, D);
            bool ok = mbar_wait(q_full, 0, 0x521u);
            auto issue_s = [&](int j) {
                const int s = j % STAGES, b = j & 1;
                if (!mbar_wait(&kv_full[s], static_cast<uint32_t>((j / STAGES) & 1), 0x522u)) return false;
                if (j >= 2 && !mbar_wait(&s_empty[b], static_cast<uint32_t>(((j >> 1) - 1) & 1), 0x523u)) return false;
                tc_fence_after();
                const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK + s * K_BYTES);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {  // K = 128 dims: 2 column blocks x 4 steps of 16
                    const int cb = ks >> 2, kk = ks & 3;
                    tc_mma_bf16(tmem + TMEM_S + static_cast<uint32_t>(BN) * b, sdesc_kmajor_sw128(q_base + cb * (Q_BYTES / 2) + 32 * kk),
                                sdesc_kmajor_sw128(k_base + cb * (K_BYTES / 2) + 32 * kk), id_s, ks > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[b]);
                return true;
            };
            if (ok && n_tiles > 0) ok = issue_s(0);
            for (int j = 0; ok && j < n_tiles; ++j) {
                if (j + 1 < n_tiles && !issue_s(j + 1)) {
                    ok = false;
                    break;
                }
                const int b = j & 1, s = j % STAGES;
                // P_j written (and, where a row's reference maximum moved, that row of O rescaled)
                if (!mbar_wait(&p_full[b], static_cast<uint32_t>((j >> 1) & 1), 0x524u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t p_base = smem_u32(sP + b * P_BYTES), v_base = smem_u32(sV + s * V_BYTES);
#pragma unroll
                for (int ks = 0; ks < BN / 16; ++ks) {  // K = BN keys: KB column blocks x 4 steps of 16
                    const int kb = ks >> 2, kk = ks & 3;
                    tc_mma_bf16(tmem + TMEM_O, sdesc_kmajor_sw128(p_base + kb * CB_BYTES + 32 * kk),
                                sdesc_kmajor_sw128(v_base + kb * CB_BYTES + 32 * kk), id_o, (j > 0 || ks > 0) ? 1u : 0u);
                }
                tc_commit(&o_done[b]);
                tc_commit(&kv_empty[s]);
            }
            tc_commit(drain);
            mbar_wait(drain, 0, 0x526u);
        }
    } else {
        // ---------------------------------------------------------------- softmax (warps 2..5)
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // query row of this thread = tensor-memory lane
        const int row = q0 + r;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const float sc = p.scale_log2;
        float m_ref = -INFINITY, l_run = 0.0f;  // reference maximum (scaled, log2 units), running sum
        bool ok = true;
        auto wait_o = [&](int i) {  // O += P_i V_i finished
            return __all_sync(0xFFFFFFFFu,
                              mbar_wait(&o_done[i & 1], static_cast<uint32_t>((i >> 1) & 1), 0x532u));
        };
        for (int j = 0; ok && j < n_tiles; ++j) {
            const int b = j & 1;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s_full[b], static_cast<uint32_t>((j >> 1) & 1), 0x531u));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                tmem_ld_32x32b_x32(t_lane + TMEM_S + static_cast<uint32_t>(BN) * b + 32u * c,
                                   *reinterpret_cast<uint32_t(*)[32]>(sv + 32 * c));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[b]);
            // causal mask (only tiles reaching past the block's first query can hide keys)
            const bool diag = (j + 1) * BN - 1 > q0;
            float mt = -INFINITY;
#pragma unroll
            for (int e = 0; e < BN; ++e) {
                if (diag && j * BN + e > row) sv[e] = __float_as_uint(-INFINITY);
                mt = fmaxf(mt, __uint_as_float(sv[e]));
            }
            mt *= sc;  // the row's maximum of this tile, scaled (finite on tile 0: key 0 is visible)
            const bool grow = mt > m_ref + TAU;
            if (j == 0) {
                m_ref = mt;
            } else if (__any_sync(0xFFFFFFFFu, grow)) {
                // rows whose maximum moved: rescale their row of O once O += P_{j-1} V_{j-1} is done
                const float f = grow ? ex2_approx(m_ref - mt) : 1.0f;
                ok = wait_o(j - 1);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_lane + TMEM_O + 32u * c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
                    tmem_st_32x32b_x32(t_lane + TMEM_O + 32u * c, v);
                }
                tmem_st_wait_att();
                tc_fence_before();
                l_run *= f;
                if (grow) m_ref = mt;
            }
            // P_j = 2^(S * scale - m_ref) <= 2^TAU, into shared-memory buffer b once O += P_{j-2} V_{j-2} read it
            float sum = 0.0f;
            uint32_t pw[BN / 2];
#pragma unroll
            for (int e = 0; e < BN / 2; ++e) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * e]), sc, -m_ref));
                const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * e + 1]), sc, -m_ref));
                sum += p0 + p1;
                pw[e] = pack_bf16x2(p0, p1);
            }
            l_run += sum;
            if (j >= 2) {
                ok = wait_o(j - 2);
                if (!ok) break;
            }
            // row r: BN bf16 = BN / 8 chunks of 16 bytes over KB column blocks; chunk cc of a
            // block at slot cc ^ (r & 7) (128-byte swizzle)
            const uint32_t prow = smem_u32(sP + b * P_BYTES) + static_cast<uint32_t>(r) * 128u;
#pragma unroll
            for (int c = 0; c < BN / 8; ++c)
                st_shared_v4(prow + static_cast<uint32_t>((c >> 3) * CB_BYTES) +
                                 (((static_cast<uint32_t>(c) & 7u) ^ (static_cast<uint32_t>(r) & 7u)) << 4),
                             pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
            fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[b]);
        }
        if (ok && n_tiles > 0) ok = wait_o(n_tiles - 1);
        if (ok) {
            tc_fence_after();
            const float inv = 1.0f / l_run;
            uint4* dst = reinterpret_cast<uint4*>(p.o + static_cast<size_t>(row) * p.ldo + h * D);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_lane + TMEM_O + 32u * c, v);
                tmem_ld_wait();
                if (row < p.M) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[4 * c + q] = make_uint4(
                            pack_bf16x2(__uint_as_float(v[8 * q]) * inv, __uint_as_float(v[8 * q + 1]) * inv),
                            pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv),
                            pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv),
                            pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace serq
