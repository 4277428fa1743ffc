/*
 * serq.h — C ABI of the SERQ W4A4 linear for NVIDIA B200 (sm_100a).
 *
 * SERQ ("Saliency-Aware Low-Rank Error Reconstruction for LLM Quantization",
 * arXiv 2603.08185) runs a W4A4 linear layer as
 *
 *     Y ~= X^_q . W^_q  +  X~_{s,q} . Q(R)
 *
 * ("量化推理" formula of the dihengye.cn reading notes, Stage 2), where
 *   - W^ = P . diag(s) . W is the weight after static activation flattening
 *     (Stage 1, SAF) and the saliency row permutation P (Stage 2);
 *   - R = W~_s - Q(W~_s) is the quantization error of the r salient rows of W^
 *     (Stage 2, single-matrix compensation), itself quantized to 4 bits
 *     (gist.science/zh summary, 2.2: "矩阵 R 本身也被量化为 4 位");
 *   - X^ = X . diag(s)^-1 . P^T is produced directly by the previous layer,
 *     into which 1/s and P are folded offline (Stage 3);
 *   - X~_s = X^[:, :r] is the salient activation slice, quantized under its
 *     own scale.
 *
 * Formats (gist.science/zh, 3: "INT4 或 MXFP4"):
 *   SERQ_FMT_INT4  : symmetric INT4 codes in [-7, 7] (s = max|x| / 7, the
 *                    "基础量化" formula with n = 4), fp32 scales: per token for
 *                    activations, per output channel for W^ and R.
 *   SERQ_FMT_MXFP4 : E2M1 codes with one E8M0 exponent per 32 consecutive
 *                    elements along the reduction axis (OCP MX v1.0).
 *   SERQ_FMT_W4A8  : the W4A8 setting of the arXiv abstract (fugumt.com): the
 *                    weight side exactly as SERQ_FMT_INT4 (W^_q and Q(R) INT4
 *                    per output channel); activations and the salient slice
 *                    INT8 per token, s = max|x| / 127 (n = 8 in "基础量化"),
 *                    codes in [-127, 127], one byte each (not packed).
 *
 * Conventions
 *   - Matrices are row-major. W is K x N (input channels x output channels,
 *     the math layout of Y = X W). Activations are M x K (tokens x channels).
 *   - 4-bit codes are packed two per byte along K: element 2j in the low
 *     nibble, 2j+1 in the high nibble. INT4 codes are two's complement.
 *     E2M1 codes are 0..15 (bit 3 = sign). E8M0 bytes are E + 127.
 *   - MXFP4 scale bytes are stored in "atoms" of 128 rows x 4 blocks (512 B):
 *     byte (row, block) of a tensor with nblk blocks per row lives at
 *         ((row / 128) * ceil(nblk / 4) + block / 4) * 512
 *           + (row % 32) * 16 + ((row % 128) / 32) * 4 + block % 4
 *     which is the layout the tensor cores read scale factors in.
 *   - The residual width is padded: rp = round_up(r, 64) (0 when r = 0).
 *     Packed salient/residual rows have rp/2 bytes; codes past r are 0.
 *   - All device pointers must be 16-byte aligned. Calls that take a
 *     stream are asynchronous on it unless stated otherwise; pass NULL for
 *     the legacy default stream.
 *   - Errors are returned as serq_status; nothing aborts or throws across
 *     the ABI. serq_last_error() gives a message for the calling thread.
 *   - The library owns serq_weight and its device buffers; the caller owns
 *     every other buffer.
 */
#ifndef SERQ_H
#define SERQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* serq_stream; /* a cudaStream_t */

typedef enum {
    SERQ_OK = 0,
    SERQ_EINVAL = 1,       /* bad argument: shape, pointer, alignment, format */
    SERQ_EUNSUPPORTED = 2, /* device is not sm_100 or shape outside the kernels' range */
    SERQ_ENOMEM = 3,       /* device allocation of a prepared weight failed */
    SERQ_ECUDA = 4,        /* a CUDA runtime call failed */
    SERQ_ETIMEOUT = 5      /* a kernel gave up waiting on a pipeline barrier */
} serq_status;

typedef enum { SERQ_FMT_INT4 = 0, SERQ_FMT_MXFP4 = 1, SERQ_FMT_W4A8 = 2 } serq_format;

typedef struct serq_weight serq_weight; /* opaque prepared linear */

/* ------------------------------------------------------------------------
 * Calibration helper.
 * Column absmax a_j = max_t |X[t, j]| of bf16 activations X (M x K, device),
 * written to absmax (K floats, device). Feeds serq_prepare_desc.act_absmax
 * (Stage 1: the SAF scales are set from calibration activations).
 * Errors: EINVAL for M < 1, K < 1, NULL or unaligned pointers.
 * ------------------------------------------------------------------------ */
serq_status serq_calib_absmax(const void* X, int M, int K, float* absmax, serq_stream stream);

/* ------------------------------------------------------------------------
 * Offline preparation (Stages 1-3 of the reading notes; gist.science/zh 2.1-2.3).
 *
 *   s_j  = sqrt(a_j / max_n |W[j, n]|)   (s_j = 1 if either is 0), unless s is given
 *   perm = channels sorted by s descending (ties: lower index first)
 *   W^   = P diag(s) W;  W^_q = RTN quantization of W^ (INT4 per output channel,
 *          MXFP4 per 32 along K)
 *   R    = W^[:r] - deq(W^_q)[:r];  Q(R) = INT4 per output channel / MXFP4 per 32 along r
 *
 * Inputs (device): W bf16 K x N; act_absmax fp32[K] or s fp32[K] (exactly one
 * non-NULL). Requirements: K % 128 == 0, N % 128 == 0, 0 <= r <= K.
 * On success *out owns device copies of perm, s, 1/s[perm], W^_q, Q(R) and
 * their scales (MXFP4: also a second, internal copy of both scale arrays in
 * the layout the prefill kernel copies into tensor memory, 4x the scale
 * bytes). Synchronizes the stream. Errors: EINVAL, EUNSUPPORTED, ENOMEM,
 * ECUDA (nothing is leaked on failure).
 * ------------------------------------------------------------------------ */
typedef struct {
    int K, N, r;
    int fmt;                  /* serq_format */
    const void* W;            /* device bf16 [K][N] */
    const float* act_absmax;  /* device fp32 [K], or NULL when s is given */
    const float* s;           /* device fp32 [K], or NULL */
    const void* R;            /* NULL (SERQ: R = W~_s - Q(W~_s)), or device bf16 [r][N]: a given
                                 matrix quantized into the residual slot instead (the second
                                 factor of the two-factor baseline, serq_linear_l2qer) */
} serq_prepare_desc;

serq_status serq_prepare(const serq_prepare_desc* desc, serq_weight** out, serq_stream stream);
void serq_weight_destroy(serq_weight* w);

/* Device views of a prepared weight (all pointers owned by the weight).
 *   perm   int32[K]   permuted position -> original channel
 *   s      fp32[K]    SAF scales, original channel order
 *   inv_s  fp32[K]    1 / s[perm[i]], permuted order (for the producer fold)
 *   wq     u8[N][K/2]         packed W^_q, K-major
 *   w_scale  INT4: fp32[N];   MXFP4: E8M0 atoms over (N rows, K/32 blocks)
 *   rq     u8[N][rp/2]        packed Q(R), r-major
 *   r_scale  INT4: fp32[N];   MXFP4: E8M0 atoms over (N rows, rp/32 blocks)   */
typedef struct {
    int K, N, r, rp, fmt;
    const int32_t* perm;
    const float* s;
    const float* inv_s;
    const uint8_t* wq;
    size_t wq_bytes;
    const void* w_scale;
    size_t w_scale_bytes;
    const uint8_t* rq;
    size_t rq_bytes;
    const void* r_scale;
    size_t r_scale_bytes;
} serq_weight_view;

serq_status serq_weight_get_view(const serq_weight* w, serq_weight_view* out);

/* ------------------------------------------------------------------------
 * The prepared weight as an artefact: export, checkpoint and import.
 *
 * SERQ's offline stages produce the permuted, flattened and quantized linear
 * once; at run time it costs nothing extra (reading notes Stage 3 and
 * gist.science/zh 2.3: the permutation and 1/s are merged into the weights
 * ahead of time). These calls move that artefact between processes and
 * devices in a canonical host form:
 *
 *   perm     int32[K]           permuted position -> original channel
 *   s        fp32[K]            SAF scales, original channel order (> 0)
 *   inv_s    fp32[K]            1 / s[perm[i]] (IEEE division), permuted order
 *   wq       u8[N][K/2]         packed W^_q (element 2j low nibble)
 *   w_scale  INT4 : fp32[N]     per output channel
 *            MXFP4: u8[N][K/32] E8M0 bytes, row-major (not the atom layout)
 *   rq       u8[N][rp/2]        packed Q(R); codes at positions >= r are 0
 *   r_scale  INT4 : fp32[N]     (zeros when r = 0)
 *            MXFP4: u8[N][rp/32] E8M0, row-major; blocks past ceil(r/32) are 0
 *
 * rp = round_up(r, 64) (0 when r = 0). The caller owns every host buffer.
 * ------------------------------------------------------------------------ */
typedef struct {
    int K, N, r, rp, fmt;
    int32_t* perm;
    float* s;
    float* inv_s;
    uint8_t* wq;
    void* w_scale;
    uint8_t* rq;
    void* r_scale;
} serq_weight_host;

/* Copy a prepared weight into canonical host buffers. dst->K..fmt are set;
 * each non-NULL pointer receives its part (NULL parts are skipped), so a
 * first call with every pointer NULL just reports the shape. Synchronizes
 * the weight's device. Errors: EINVAL (NULL w or dst), ECUDA. */
serq_status serq_weight_export(const serq_weight* w, serq_weight_host* dst);

/* Build a prepared weight on the current device from canonical host buffers
 * (all non-NULL, except rq/r_scale when r = 0): for example one exported
 * from another process, read from a checkpoint, or quantized by other
 * tooling in this layout. The content is checked first: shape rules as for
 * serq_prepare, rp = round_up(r, 64), perm a permutation of 0..K-1, s finite
 * and > 0, inv_s[i] == 1/s[perm[i]] bit for bit, INT4 codes in [-7, 7] and
 * scales finite and >= 0, no E8M0 byte 0xFF, zero codes / scale blocks past
 * r. The result is bit-identical on export to the buffers it was built from.
 * Synchronizes the stream. Errors: EINVAL (content), EUNSUPPORTED, ENOMEM,
 * ECUDA; nothing is leaked on failure. */
serq_status serq_weight_create_from_host(const serq_weight_host* src, serq_weight** out, serq_stream stream);

/* Checkpoint file: a 64-byte header (magic "SERQWGT", version 1, fmt, K, N,
 * r, rp, payload size, FNV-1a-64 checksum of the payload) followed by the
 * canonical parts above in their listed order, little-endian.
 *   serq_weight_save: export + write (synchronizes the weight's device).
 *   serq_weight_load: read + check (header, size, checksum, content) +
 *     serq_weight_create_from_host on the current device.
 *   serq_weight_file_write / serq_weight_file_read: the same file from / to
 *     host buffers, without a GPU. file_read sets dst->K..fmt and fills the
 *     non-NULL pointers (a first call with every pointer NULL reports the
 *     shape so the caller can size its buffers).
 * Errors: EINVAL (NULL arguments, unreadable / unwritable / truncated /
 * corrupt file, content), plus those of the device calls. */
serq_status serq_weight_save(const serq_weight* w, const char* path);
serq_status serq_weight_load(const char* path, serq_weight** out, serq_stream stream);
serq_status serq_weight_file_write(const char* path, const serq_weight_host* src);
serq_status serq_weight_file_read(const char* path, serq_weight_host* dst);

/* Test hook (no counterpart in the paper): the next n device allocations of a
 * prepared weight (serq_prepare, serq_weight_create_from_host,
 * serq_weight_load) fail with SERQ_ENOMEM without calling cudaMalloc, so the
 * out-of-memory path can be tested without exhausting the GPU. n = 0 clears
 * it. Returns the previous count. */
int serq_debug_fail_next_allocations(int n);

/* ------------------------------------------------------------------------
 * Producer fold (Stage 3: "行/列排列离线合并到权重中"; gist.science/zh 2.3).
 * dst[row][i] = bf16(src[row][perm[i]] / s[perm[i]]) for a row-major bf16
 * matrix whose K columns are this layer's input channels: the producer's
 * weight (then X_prev . dst = X^), or an activation block (then dst = X^).
 * src, dst: device, rows x K, must not overlap. Errors: EINVAL.
 * ------------------------------------------------------------------------ */
serq_status serq_fold_producer(const serq_weight* w, const void* src, int rows, void* dst,
                               serq_stream stream);

/* ------------------------------------------------------------------------
 * Runtime activation quantization ("基础量化" per token; X~_{s,q} of "量化推理").
 *
 * Xhat: device bf16 [M][K]. Outputs (device, caller-allocated; sizes from
 * serq_act_buffer_sizes):
 *   INT4 : xq u8[M][K/2], xs fp32[M] (= max_i|x|/7), xsq u8[M][rp/2], xss fp32[M]
 *          (= max_{i<r}|x|/7); codes rne(x / s) clipped to [-7, 7].
 *   W4A8 : xq s8[M][K], xs fp32[M] (= max_i|x|/127), xsq s8[M][rp], xss fp32[M]
 *          (= max_{i<r}|x|/127); codes rne(x / s) clipped to [-127, 127].
 *   MXFP4: xq u8[M][K/2], xs E8M0 atoms (M rows, K/32 blocks), xsq u8[M][rp/2],
 *          xss E8M0 atoms (M rows, rp/32 blocks; the slice's own blocks over
 *          its first r columns, a short last block padded with zeros).
 *   Scale bytes of atom rows >= M are not written.
 * xsq/xss may be NULL when r == 0. Requirements: K % 128 == 0, 0 <= r <= K.
 * Errors: EINVAL.
 * ------------------------------------------------------------------------ */
typedef struct {
    size_t xq, xs, xsq, xss;
} serq_act_sizes;

serq_status serq_act_buffer_sizes(int M, int K, int r, int fmt, serq_act_sizes* out);
serq_status serq_quant_act(const void* Xhat, int M, int K, int r, int fmt, void* xq, void* xs,
                           void* xsq, void* xss, serq_stream stream);

/* ------------------------------------------------------------------------
 * Producers with the fold and the activation quantization fused (reading
 * notes Stage 3, gist.science/zh 2.3: the permutation and 1/s are merged into
 * the layer that produces the linear's input). One pass reads the producer's
 * input and writes serq_quant_act's outputs for X^ (same layouts, same
 * sizes: serq_act_buffer_sizes(M, w->K, w->r, w->fmt)); X^ itself is not
 * stored unless `xhat` (bf16 [M][K], may be NULL) asks for a copy.
 * w is the consuming linear (its perm, 1/s[perm], K, r and format).
 *
 * serq_rmsnorm_quant_act: H bf16 [M][K] (original channel order), gamma bf16
 *   [K], eps >= 0:
 *     rstd[m] = 1 / sqrt(fp32(sum_j H[m,j]^2) / K + eps)
 *     X^[m,i] = bf16(fp32(H[m, perm[i]] * rstd[m]) * fp32(gamma[perm[i]] * inv_s[i]))
 *   Every step is one IEEE fp32 rounding; the sum of squares is accumulated
 *   in fp64 and rounded once. RMSNorm is the producer of q/k/v and gate/up.
 * serq_swiglu_quant_act: Ygu bf16 [M][2K] = [gate | up] outputs (original
 *   channel order):
 *     X^[m,i] = bf16(fp32(fp32(silu(g) * u) * inv_s[i])), g = Ygu[m, perm[i]],
 *     u = Ygu[m, K + perm[i]], silu(g) = g / (1 + expf(-g)) in fp32.
 *   SwiGLU is the producer of down.
 * Requirements: M >= 1, K <= 32768, 16-byte aligned pointers. Asynchronous.
 * Errors: EINVAL, EUNSUPPORTED, ECUDA.
 * ------------------------------------------------------------------------ */
serq_status serq_rmsnorm_quant_act(const serq_weight* w, const void* H, const void* gamma, float eps, int M,
                                   void* xq, void* xs, void* xsq, void* xss, void* xhat, serq_stream stream);
serq_status serq_swiglu_quant_act(const serq_weight* w, const void* Ygu, int M, void* xq, void* xs, void* xsq,
                                  void* xss, void* xhat, serq_stream stream);

/* ------------------------------------------------------------------------
 * The SwiGLU producer fused into the gate/up linear's epilogue (MXFP4 only).
 *
 * serq_prepare_swiglu: `gate_up` describes [W_gate | W_up] (K x 2F, bf16,
 *   device; SAF scales and rank of the gate/up linear as in serq_prepare),
 *   `down` is the prepared down linear (K = F) it feeds. The down linear's
 *   input permutation is merged into the gate/up weight's output columns
 *   (Stage 3: "行/列排列离线合并到权重中"): column block t of 256 holds the
 *   gate then the up columns of down's permuted input positions 128 t ..
 *   128 t + 127. The weight keeps a copy of down's 1/s[perm] (F floats).
 *   Quantization per output channel is unaffected by the arrangement.
 *   Synchronizes. Errors: EINVAL, EUNSUPPORTED (not MXFP4), ENOMEM, ECUDA.
 * serq_linear_swiglu_quant: the gate/up linear for M > 128 (CTA-pair
 *   kernel) whose epilogue, instead of writing Y, computes for each row m and
 *   permuted down channel i
 *       X^_d[m,i] = bf16(fp32(fp32(silu(g) * u) * inv_s_d[i])),
 *       silu(g) = g / (1 + exp(-g)) with the fast fp32 exponential and
 *       division (a few ulp; X^_d is rounded to bf16 right after), g, u the
 *       fp32 accumulators,
 *   and writes serq_quant_act's MXFP4 outputs for X^_d with down's rank:
 *   hq/hs/hsq/hss sized by serq_act_buffer_sizes(M, F, down r, MXFP4).
 *   xhat: NULL, or bf16 [M][F] receiving X^_d. xq..xss are gate/up's input
 *   (serq_quant_act of its X^). M <= 128 returns EUNSUPPORTED (use
 *   serq_linear and serq_swiglu_quant_act with an unarranged gate/up).
 * ------------------------------------------------------------------------ */
serq_status serq_prepare_swiglu(const serq_prepare_desc* gate_up, const serq_weight* down, serq_weight** out,
                                serq_stream stream);
serq_status serq_linear_swiglu_quant(const serq_weight* w, int M, const void* xq, const void* xs, const void* xsq,
                                     const void* xss, void* hq, void* hs, void* hsq, void* hss, void* xhat,
                                     serq_stream stream);

/* ------------------------------------------------------------------------
 * The plain fold fused with the quantization, for a producer that cannot
 * fold the permutation and 1/s into itself (the attention output feeding the
 * o projection): X^[m,i] = bf16(X[m, perm[i]] / s[perm[i]]) (serq_fold_producer's
 * arithmetic), then serq_quant_act's outputs for X^, in one pass. X: bf16
 * [M][w->K]. xhat: NULL or a bf16 [M][K] copy of X^. Errors as above.
 * ------------------------------------------------------------------------ */
serq_status serq_fold_quant_act(const serq_weight* w, const void* X, int M, void* xq, void* xs, void* xsq, void* xss,
                                void* xhat, serq_stream stream);

/* ------------------------------------------------------------------------
 * The LLaMA block around the SERQ linears (for the 2K-prefill time to first
 * token the reading notes report under "GPU 性能分析"); standard definitions,
 * bf16 storage, fp32 arithmetic.
 *
 * serq_rope: in place, rotate-half rotary embedding of heads [0, n_heads) of a
 *   token-major bf16 matrix x (row stride ld elements, head h at columns
 *   [h*head_dim, +head_dim)): for pair i < head_dim/2 at position pos0 + m,
 *   angle = (pos0 + m) * base^(-2i/head_dim),
 *   (x_i, x_{i+d/2}) <- (x_i cos - x_{i+d/2} sin, x_{i+d/2} cos + x_i sin).
 * serq_attention_prefill: causal grouped-query attention, head_dim 128:
 *   O_h = softmax(Q_h K_g^T / sqrt(128) + mask(key > query)) V_g,
 *   g = h / (n_q / n_kv); q [M][ldq] (heads at column h*128), k, v [M][ldkv],
 *   o [M][ldo]; all bf16, 16-byte aligned, leading dimensions multiples of 8.
 *   tcgen05 bf16 MMAs with fp32 accumulation in tensor memory and an online
 *   softmax (the scores never reach global memory); V is first transposed
 *   into stream-ordered device scratch (n_kv * 128 * round_up(M, 64) bf16,
 *   allocated and freed on `stream` from a memory pool of the library's that
 *   keeps what it has grown to).
 * serq_add: out = bf16(a + b) elementwise over n bf16 values (n % 8 == 0).
 * All asynchronous on `stream`. Errors: EINVAL, EUNSUPPORTED (head_dim), ECUDA.
 * ------------------------------------------------------------------------ */
serq_status serq_rope(void* x, int M, int ld, int n_heads, int head_dim, float base, int pos0, serq_stream stream);
serq_status serq_attention_prefill(const void* q, int ldq, const void* k, const void* v, int ldkv, int M, int n_q,
                                   int n_kv, int head_dim, void* o, int ldo, serq_stream stream);
serq_status serq_add(const void* a, const void* b, void* out, size_t n, serq_stream stream);

/* ------------------------------------------------------------------------
 * The SERQ linear (the "量化推理" formula): one kernel launch computing
 *   MXFP4: Y = bf16( sum over K of X^_q W^_q  +  sum over r of X~_{s,q} Q(R) ),
 *          both block-scaled products accumulated into one fp32 tile;
 *   INT4, W4A8 : acc1 = sum_i qx qw, acc2 = sum_{i<r} qxs qR (int32, exact),
 *          Y = bf16(acc1 * xs[m] * w_scale[n] + acc2 * xss[m] * r_scale[n]).
 * Inputs are serq_quant_act's outputs for the same (M, K, r, fmt).
 * Y: device bf16 [M][N]. acc_dbg: NULL, or (INT4 weights: INT4, W4A8) device int32
 * [2][M][N] receiving acc1 and acc2.
 * Kernels (MXFP4): M <= 16 a split-K weight-streaming kernel (its split CTAs
 * form a thread-block cluster; launched with programmatic dependent launch,
 * so it may start streaming weights while the preceding kernel of the stream
 * finishes, and reads xq/xs and writes Y only after it completes);
 * 16 < M <= 128 a one-CTA tensor-core kernel; M > 128 a CTA-pair kernel.
 * INT4 and W4A8: one tensor-core kernel for every M (W4A8 loads the int8
 * activations straight into the MMA layout). Results do not depend on which
 * kernel ran beyond fp32 summation order (MXFP4); INT4 accumulators are exact.
 * Errors: EINVAL (shape/format mismatch with w, NULL/unaligned pointers),
 * EUNSUPPORTED (not an sm_100 device).
 * ------------------------------------------------------------------------ */
serq_status serq_linear(const serq_weight* w, int M, const void* xq, const void* xs,
                        const void* xsq, const void* xss, void* Y, int32_t* acc_dbg,
                        serq_stream stream);

/* ------------------------------------------------------------------------
 * The two-factor baseline SERQ is compared against (L2QER; reading notes
 * "L2QER 的双矩阵路径", gist.science/pt 1):
 *     Y = X_q W_q + Q(X_q L_{1,q}) L_{2,q}
 * Three launches, in order on `stream`: T = serq_linear(l1, X_q) (bf16
 * [M][k] in the caller's scratch T), serq_quant_act(T, r = k) into tq/ts/
 * tsq/tss (sizes serq_act_buffer_sizes(M, k, k, fmt)), then
 * serq_linear(main, X_q, Q(T)) with Q(T) as the residual operand.
 *   main: serq_prepare of W with desc.R = L2 (k x N) and r = k;
 *   l1  : serq_prepare of L1 (K x k) with r = 0 and desc.s = main's SAF scales
 *         (so L1 is folded with main's permutation and 1/s);
 *   xq/xs: serq_quant_act(X^, r = 0) for main's K and format.
 * k must meet serq_quant_act's rules (k % 128 == 0). Errors: those of the
 * three calls, EINVAL for mismatched weights.
 * ------------------------------------------------------------------------ */
serq_status serq_linear_l2qer(const serq_weight* main, const serq_weight* l1, int M, const void* xq, const void* xs,
                              void* T, void* tq, void* ts, void* tsq, void* tss, void* Y, serq_stream stream);

/* ------------------------------------------------------------------------
 * serq_linear_small_m_noalloc — the small-M (M <= 16) MXFP4 linear for
 * callers that cannot allocate device memory. (The SERQ paper has no
 * counterpart; this is an interface addition of this library.)
 *
 * Who needs it: runtimes that plan every device buffer ahead of time and do
 * not allow cudaMalloc on the serving path (cudaMalloc can synchronize the
 * device and can fail under memory pressure), and code that holds packed
 * weights in memory it manages itself rather than in a serq_weight. Such a
 * caller passes every input and the output as raw device pointers; the call
 * allocates nothing (no cudaMalloc/cudaFree, no allocating library routine).
 *
 * Inputs, in the layouts of include/serq.h (for example the buffers that
 * serq_weight_get_view returns for an MXFP4 weight, and serq_quant_act's
 * outputs for the same M, K, r): wq u8[N][K/2], w_scale E8M0 atoms
 * (N rows, K/32 blocks), rq u8[N][rp/2], r_scale E8M0 atoms (N rows, rp/32
 * blocks), xq/xs/xsq/xss. rq, r_scale, xsq and xss may be NULL when r == 0.
 * Output: Y bf16 [M][N]. Same result as serq_linear for the same operands.
 *
 * Scratch: the split-K partial sums and tickets of the small-M kernel live
 * in one static device array of 4 MiB inside the library (held by every GPU
 * that loads the library until the process exits). Limits: 1 <= M <= 16,
 * N <= 131072 (the ticket area) and M*N <= 1047552 (the partial-sum area);
 * larger sizes return SERQ_EINVAL with the limit in serq_last_error(). The
 * number of K splits shrinks when M*N leaves room for fewer.
 * Every call shares the array and it keeps the last call's contents (each
 * call clears the tickets it uses, on `stream`, before its kernel): calls
 * that overlap on the GPU (other streams, other host threads) race.
 * The first call on a device does a one-time set-up (it looks up the
 * array's device address with cudaGetSymbolAddress); make that first call
 * before any stream capture. Asynchronous on `stream`.
 * Errors: EINVAL, EUNSUPPORTED, ECUDA.
 * ------------------------------------------------------------------------ */
serq_status serq_linear_small_m_noalloc(int M, int K, int N, int r, const void* wq, const void* w_scale,
                                        const void* rq, const void* r_scale, const void* xq, const void* xs,
                                        const void* xsq, const void* xss, void* Y, serq_stream stream);

/* Synchronizes the stream, then reports (and clears) any device-side pipeline
 * timeout recorded by this library's kernels on the current device:
 * SERQ_ETIMEOUT if one occurred since the last call, else SERQ_OK
 * (SERQ_ECUDA if the stream itself failed). */
serq_status serq_device_status(serq_stream stream);

/* ---------------------------------------------------------------------------
 * serq_selftest_wait -- exercise the bounded pipeline wait (the pages have no
 * counterpart; it exists so the timeout path can be tested on a GPU without
 * stalling a real pipeline).
 * One single-CTA kernel initialises an mbarrier expecting one arrival and
 * waits for its first phase with the same bounded wait the GEMM pipelines use,
 * but with a limit of `limit_cycles` SM clock cycles (1 .. 4e9). If `arrive`
 * is non-zero the barrier is completed first and the wait returns at once;
 * otherwise nothing completes it, the wait runs out after `limit_cycles`, and
 * the kernel records site 0xF01 and returns: the next serq_device_status()
 * reports SERQ_ETIMEOUT and clears the record. The CUDA context stays usable
 * either way. Asynchronous on `stream`. Errors: EINVAL, ECUDA.
 * ------------------------------------------------------------------------ */
serq_status serq_selftest_wait(long long limit_cycles, int arrive, serq_stream stream);

const char* serq_last_error(void); /* thread-local message of the last failure */
const char* serq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SERQ_H */
