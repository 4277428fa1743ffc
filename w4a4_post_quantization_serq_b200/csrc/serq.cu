// C ABI of the SERQ W4A4 linear (include/serq.h): argument checks, device
// buffers of prepared weights, tensor-map encoding and kernel launches.
// The kernels themselves live in the *.cuh files of this directory; this is
// the only translation unit, so they share one device-side timeout flag.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "serq.h"

#include "ptx.cuh"
#include "quant_act.cuh"
#include "prepare.cuh"
#include "gemm_mxfp4.cuh"
#include "gemm_int4.cuh"
#include "gemm_mxfp4_decode.cuh"
#include "gemm_mxfp4_pair.cuh"

using namespace serq;

// ============================================================== errors
namespace {

thread_local std::string g_last_error;

serq_status fail(serq_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

serq_status cuda_fail(cudaError_t e, const char* what) {
    return fail(SERQ_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define SERQ_CUDA(call)                                   \
    do {                                                  \
        cudaError_t e_ = (call);                          \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int round_up(int x, int m) { return (x + m - 1) / m * m; }

int residual_width(int r) { return r > 0 ? round_up(r, 64) : 0; }

size_t atom_bytes(int rows, int blocks) {
    return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((blocks + 3) / 4) * 512u;
}

// ============================================================== device info
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int ok = -1;  // -1 unknown, 0 unsupported, 1 sm_100
    int sms = 0;
    bool smem_set_mx = false;
    bool smem_set_i4 = false;
    bool smem_set_mxd = false;
    bool smem_set_mxp = false;
    int pair_clusters = 0;  // co-resident 2-CTA clusters of the pair kernel
};

// split-K ranges of the small-M kernel. Two CTAs fit per SM. A launch first
// takes one CTA per SM, leaving the other slot to the next launch, whose CTAs
// then prefetch their weight stages while this one finishes; when a CTA
// would still have more K-tiles than its ring holds, the launch takes both
// slots instead (more bytes in flight). At most kMaxDecodeSplits (the
// portable cluster size), never more than the K-tiles.
constexpr int kMaxDecodeSplits = mxd::MAX_SPLITS;
constexpr int kMaxDecodeTokens = 16;

int decode_splits(int n_blocks, int k_tiles, int sms) {
    auto fit = [&](int slots) {
        int s = slots / n_blocks;
        if (s > kMaxDecodeSplits) s = kMaxDecodeSplits;
        if (s > k_tiles) s = k_tiles;
        return s < 1 ? 1 : s;
    };
    const int s1 = fit(sms);
    return (k_tiles + s1 - 1) / s1 > mxd::STAGES ? fit(2 * sms) : s1;
}

// One-time per-device set-up of both forms of the small-M kernel.
serq_status decode_setup(DeviceInfo* info) {
    if (info->smem_set_mxd) return SERQ_OK;
    SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   mxd::SMEM_BYTES));
    SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_decode_kernel<false>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, mxd::SMEM_BYTES));
    // all of the unified L1/shared storage as shared memory, so that two CTAs fit per SM
    SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_decode_kernel<true>,
                                   cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared));
    SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_decode_kernel<false>,
                                   cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared));
    info->smem_set_mxd = true;
    return SERQ_OK;
}
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

serq_status device_check(int* dev_out, DeviceInfo** info_out) {
    int dev = 0;
    SERQ_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(SERQ_EUNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (d.ok < 0) {
        int major = 0, minor = 0;
        SERQ_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
        SERQ_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
        SERQ_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        d.ok = (major == 10 && minor == 0) ? 1 : 0;
    }
    if (d.ok != 1) return fail(SERQ_EUNSUPPORTED, "device %d is not an sm_100 (B200-class) GPU", dev);
    *dev_out = dev;
    *info_out = &d;
    return SERQ_OK;
}

// ============================================================== tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D uint8 tensor of `rows` rows of `inner` bytes; boxes of box_inner x box_rows.
serq_status make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                     uint32_t box_rows, bool swizzle128);

// MXFP4 scale-atom array (a multiple of 512 B) as rows of 256 B; a box is two
// atoms (256 x 4). Rows past the end read as zeros.
serq_status make_scale_map(CUtensorMap* map, const void* base, size_t bytes) {
    return make_map(map, base, 256, bytes / 256, 256, 4, false);
}

serq_status make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                     uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return fail(SERQ_ECUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SERQ_ECUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return SERQ_OK;
}

// box geometry per format: MXFP4 loads 128-byte swizzled rows straight into
// the MMA layout; INT4 loads 64 packed bytes per row into staging.
uint32_t box_inner_bytes(int fmt) { return fmt == SERQ_FMT_MXFP4 ? 128u : 64u; }

}  // namespace

// ============================================================== weight handle
struct serq_weight {
    int K, N, r, rp, fmt, device;
    void* arena;
    int32_t* perm;
    float* s;
    float* s_perm;
    float* inv_s;
    uint8_t* wq;
    size_t wq_bytes;
    void* wsc;
    size_t wsc_bytes;
    uint8_t* rq;
    size_t rq_bytes;
    void* rsc;
    size_t rsc_bytes;
    uint8_t* wscw;         // MXFP4 weight / residual scales in the wide layout of the CTA-pair kernel
    size_t wscw_bytes;
    uint8_t* rscw;
    size_t rscw_bytes;
    CUtensorMap tm_w;      // B operand of the prefill kernels (256-row boxes)
    CUtensorMap tm_r;
    CUtensorMap tm_w128;   // A operand of the small-M kernel (128-row boxes, MXFP4)
    CUtensorMap tm_r128;
    CUtensorMap tm_wsf;    // wide MXFP4 scales as 256 B rows (box: two 4 KB atom pairs)
    CUtensorMap tm_rsf;
};

// ============================================================== allocation-free small-M entry
// Scratch of serq_linear_small_m_noalloc: split-K tickets (first 4 KiB, one
// uint32 per 128 output channels) followed by fp32 partial sums. It lives in
// the library image, so every GPU that loads the library holds it until exit.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr size_t kNoAllocTicketBytes = 4096;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, looked up once
// per device (host code only holds a stand-in symbol, not a device address).
serq_status noalloc_scratch(int dev, void** out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SERQ_OK;
}
}  // namespace

// One bounded mbarrier wait, completed first or left to run out (site 0xF01).
__global__ void wait_selftest_kernel(long long limit_cycles, int arrive) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (arrive) mbar_arrive(&bar);
        mbar_wait_limit(&bar, 0u, 0xF01u, limit_cycles);
    }
}

extern "C" {

const char* serq_last_error(void) { return g_last_error.c_str(); }

const char* serq_version(void) { return "serq-b200 0.1 (sm_100a)"; }

serq_status serq_act_buffer_sizes(int M, int K, int r, int fmt, serq_act_sizes* out) {
    if (out == nullptr) return fail(SERQ_EINVAL, "out is NULL");
    if (M < 1 || K < 128 || K % 128 != 0 || r < 0 || r > K)
        return fail(SERQ_EINVAL, "bad shape M=%d K=%d r=%d (need M>=1, K%%128==0, 0<=r<=K)", M, K, r);
    if (fmt != SERQ_FMT_INT4 && fmt != SERQ_FMT_MXFP4) return fail(SERQ_EINVAL, "unknown format %d", fmt);
    const int rp = residual_width(r);
    out->xq = static_cast<size_t>(M) * (K / 2);
    out->xsq = static_cast<size_t>(M) * (rp / 2);
    if (fmt == SERQ_FMT_INT4) {
        out->xs = static_cast<size_t>(M) * 4;
        out->xss = rp > 0 ? static_cast<size_t>(M) * 4 : 0;
    } else {
        out->xs = atom_bytes(M, K / 32);
        out->xss = rp > 0 ? atom_bytes(M, rp / 32) : 0;
    }
    return SERQ_OK;
}

serq_status serq_calib_absmax(const void* X, int M, int K, float* absmax, serq_stream stream) {
    if (X == nullptr || absmax == nullptr) return fail(SERQ_EINVAL, "NULL pointer");
    if (M < 1 || K < 1) return fail(SERQ_EINVAL, "bad shape M=%d K=%d", M, K);
    if (!aligned16(X) || !aligned16(absmax)) return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    SERQ_CUDA(cudaMemsetAsync(absmax, 0, sizeof(float) * K, s));
    const int rows = 64;
    dim3 grid((K + 255) / 256, (M + rows - 1) / rows);
    calib_absmax_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(X), M, K, rows,
                                             reinterpret_cast<unsigned int*>(absmax));
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

void serq_weight_destroy(serq_weight* w) {
    if (w == nullptr) return;
    if (w->arena != nullptr) {
        int cur = -1;
        cudaGetDevice(&cur);
        if (cur != w->device) cudaSetDevice(w->device);
        cudaFree(w->arena);
        if (cur != w->device && cur >= 0) cudaSetDevice(cur);
    }
    delete w;
}

serq_status serq_prepare(const serq_prepare_desc* desc, serq_weight** out, serq_stream stream) {
    if (desc == nullptr || out == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    *out = nullptr;
    const int K = desc->K, N = desc->N, r = desc->r, fmt = desc->fmt;
    if (K < 128 || K % 128 != 0 || K > 32768 || N < 128 || N % 128 != 0 || r < 0 || r > K)
        return fail(SERQ_EINVAL, "bad shape K=%d N=%d r=%d (need K%%128==0, K<=32768, N%%128==0, 0<=r<=K)", K, N,
                    r);
    if (fmt != SERQ_FMT_INT4 && fmt != SERQ_FMT_MXFP4) return fail(SERQ_EINVAL, "unknown format %d", fmt);
    if (desc->W == nullptr || !aligned16(desc->W)) return fail(SERQ_EINVAL, "W must be a 16-byte aligned pointer");
    if ((desc->act_absmax == nullptr) == (desc->s == nullptr))
        return fail(SERQ_EINVAL, "give exactly one of act_absmax and s");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    const int rp = residual_width(r);
    auto* w = new serq_weight();
    std::memset(w, 0, sizeof(*w));
    w->K = K;
    w->N = N;
    w->r = r;
    w->rp = rp;
    w->fmt = fmt;
    w->device = dev;
    w->wq_bytes = static_cast<size_t>(N) * (K / 2);
    w->rq_bytes = static_cast<size_t>(N) * (rp / 2);
    if (fmt == SERQ_FMT_INT4) {
        w->wsc_bytes = static_cast<size_t>(N) * 4;
        w->rsc_bytes = static_cast<size_t>(N) * 4;
    } else {
        w->wsc_bytes = atom_bytes(N, K / 32);
        w->rsc_bytes = rp > 0 ? atom_bytes(N, rp / 32) : 0;
        const size_t pairs = static_cast<size_t>((N / 128 + 1) / 2);
        w->wscw_bytes = pairs * (K / 128) * 4096;
        w->rscw_bytes = rp > 0 ? pairs * ((rp + 127) / 128) * 4096 : 0;
    }
    // one arena: perm, s, s_perm, inv_s, wq, wsc, rq, rsc, then scratch
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    const size_t o_perm = take(4u * K), o_s = take(4u * K), o_sp = take(4u * K), o_inv = take(4u * K);
    const size_t o_wq = take(w->wq_bytes), o_wsc = take(w->wsc_bytes);
    const size_t o_rq = take(w->rq_bytes), o_rsc = take(w->rsc_bytes);
    const size_t o_wscw = take(w->wscw_bytes), o_rscw = take(w->rscw_bytes);
    const size_t keep = off;
    const size_t o_b = take(4u * K), o_col = take(4u * N);
    void* arena = nullptr;
    const cudaError_t ae = cudaMalloc(&arena, off);
    if (ae != cudaSuccess) {
        delete w;
        cudaGetLastError();
        return fail(SERQ_ENOMEM, "cudaMalloc(%zu) failed: %s", off, cudaGetErrorString(ae));
    }
    (void)keep;
    uint8_t* base = static_cast<uint8_t*>(arena);
    w->arena = arena;
    w->perm = reinterpret_cast<int32_t*>(base + o_perm);
    w->s = reinterpret_cast<float*>(base + o_s);
    w->s_perm = reinterpret_cast<float*>(base + o_sp);
    w->inv_s = reinterpret_cast<float*>(base + o_inv);
    w->wq = base + o_wq;
    w->wsc = base + o_wsc;
    w->rq = base + o_rq;
    w->rsc = base + o_rsc;
    w->wscw = base + o_wscw;
    w->rscw = base + o_rscw;
    float* tmp_b = reinterpret_cast<float*>(base + o_b);
    unsigned int* tmp_col = reinterpret_cast<unsigned int*>(base + o_col);

    auto bail = [&](serq_status st) {
        cudaStreamSynchronize(cs);
        serq_weight_destroy(w);
        return st;
    };
#define PREP_CUDA(call)                                          \
    do {                                                         \
        cudaError_t e_ = (call);                                 \
        if (e_ != cudaSuccess) return bail(cuda_fail(e_, #call)); \
    } while (0)

    const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(desc->W);
    PREP_CUDA(cudaMemsetAsync(arena, 0, off, cs));
    // Stage 1: SAF scales
    if (desc->act_absmax != nullptr) {
        row_absmax_kernel<<<(K + 7) / 8, 256, 0, cs>>>(W, K, N, tmp_b);
        saf_scale_kernel<<<(K + 255) / 256, 256, 0, cs>>>(desc->act_absmax, tmp_b, K, w->s);
    } else {
        PREP_CUDA(cudaMemcpyAsync(w->s, desc->s, 4u * K, cudaMemcpyDeviceToDevice, cs));
    }
    // Stage 2: saliency order
    saliency_rank_kernel<<<(K + 255) / 256, 256, 0, cs>>>(w->s, K, w->perm, w->s_perm, w->inv_s);
    PREP_CUDA(cudaGetLastError());
    // fold + quantize W^, then the residual of the first r rows
    const dim3 qblock(32, 8);
    const dim3 qgrid(N / 32, (K / 32 + 7) / 8);
    if (fmt == SERQ_FMT_INT4) {
        const int rows = 128;
        weight_colamax_kernel<<<dim3(N / 256 + (N % 256 != 0), (K + rows - 1) / rows), 256, 0, cs>>>(W, w->s, K, N,
                                                                                                    rows, tmp_col);
        weight_quant_int4_kernel<<<qgrid, qblock, 0, cs>>>(W, w->perm, w->s_perm, tmp_col, K, N, w->wq,
                                                           static_cast<float*>(w->wsc));
        if (r > 0)
            residual_int4_kernel<<<(N + 127) / 128, 128, 0, cs>>>(W, w->perm, w->s_perm,
                                                                  static_cast<const float*>(w->wsc), N, r, rp, w->rq,
                                                                  static_cast<float*>(w->rsc));
    } else {
        weight_quant_mxfp4_kernel<<<qgrid, qblock, 0, cs>>>(W, w->perm, w->s_perm, K, N, w->wq,
                                                            static_cast<uint8_t*>(w->wsc));
        if (r > 0)
            residual_mxfp4_kernel<<<dim3(N / 32, (rp / 32 + 7) / 8), qblock, 0, cs>>>(
                W, w->perm, w->s_perm, K, N, r, rp, w->rq, static_cast<uint8_t*>(w->rsc));
        scale_widen_kernel<<<static_cast<unsigned>((w->wscw_bytes / 16 + 255) / 256), 256, 0, cs>>>(
            static_cast<const uint8_t*>(w->wsc), N / 128, K / 128, w->wscw, w->wscw_bytes);
        if (rp > 0)
            scale_widen_kernel<<<static_cast<unsigned>((w->rscw_bytes / 16 + 255) / 256), 256, 0, cs>>>(
                static_cast<const uint8_t*>(w->rsc), N / 128, (rp + 127) / 128, w->rscw, w->rscw_bytes);
    }
    PREP_CUDA(cudaGetLastError());
    PREP_CUDA(cudaStreamSynchronize(cs));

    const uint32_t bi = box_inner_bytes(fmt);
    const bool swz = fmt == SERQ_FMT_MXFP4;
    if (serq_status st = make_map(&w->tm_w, w->wq, K / 2, N, bi, 256, swz)) return bail(st);
    if (rp > 0) {
        if (serq_status st = make_map(&w->tm_r, w->rq, rp / 2, N, bi, 256, swz)) return bail(st);
    } else {
        w->tm_r = w->tm_w;
    }
    if (fmt == SERQ_FMT_MXFP4) {
        if (serq_status st = make_map(&w->tm_w128, w->wq, K / 2, N, 128, 128, true)) return bail(st);
        if (serq_status st = make_map(&w->tm_wsf, w->wscw, 256, w->wscw_bytes / 256, 256, 32, false)) return bail(st);
        if (rp > 0) {
            if (serq_status st = make_map(&w->tm_rsf, w->rscw, 256, w->rscw_bytes / 256, 256, 32, false))
                return bail(st);
        } else {
            w->tm_rsf = w->tm_wsf;
        }
        if (rp > 0) {
            if (serq_status st = make_map(&w->tm_r128, w->rq, rp / 2, N, 128, 128, true)) return bail(st);
        } else {
            w->tm_r128 = w->tm_w128;
        }
    }
#undef PREP_CUDA
    *out = w;
    return SERQ_OK;
}

serq_status serq_weight_get_view(const serq_weight* w, serq_weight_view* out) {
    if (w == nullptr || out == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    out->K = w->K;
    out->N = w->N;
    out->r = w->r;
    out->rp = w->rp;
    out->fmt = w->fmt;
    out->perm = w->perm;
    out->s = w->s;
    out->inv_s = w->inv_s;
    out->wq = w->wq;
    out->wq_bytes = w->wq_bytes;
    out->w_scale = w->wsc;
    out->w_scale_bytes = w->wsc_bytes;
    out->rq = w->rq;
    out->rq_bytes = w->rq_bytes;
    out->r_scale = w->rsc;
    out->r_scale_bytes = w->rsc_bytes;
    return SERQ_OK;
}

serq_status serq_fold_producer(const serq_weight* w, const void* src, int rows, void* dst, serq_stream stream) {
    if (w == nullptr || src == nullptr || dst == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    if (rows < 1) return fail(SERQ_EINVAL, "rows must be >= 1");
    if (!aligned16(src) || !aligned16(dst)) return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    const size_t bytes = static_cast<size_t>(rows) * w->K * 2;
    const uint8_t* a = static_cast<const uint8_t*>(src);
    const uint8_t* b = static_cast<const uint8_t*>(dst);
    if (a < b + bytes && b < a + bytes) return fail(SERQ_EINVAL, "src and dst overlap");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const size_t total = static_cast<size_t>(rows) * w->K;
    fold_producer_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, cs>>>(
        static_cast<const __nv_bfloat16*>(src), rows, w->K, w->perm, w->s_perm, static_cast<__nv_bfloat16*>(dst));
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

serq_status serq_quant_act(const void* Xhat, int M, int K, int r, int fmt, void* xq, void* xs, void* xsq, void* xss,
                           serq_stream stream) {
    serq_act_sizes sz;
    if (serq_status st = serq_act_buffer_sizes(M, K, r, fmt, &sz)) return st;
    if (K > 32768) return fail(SERQ_EUNSUPPORTED, "K=%d above the supported 32768", K);
    if (Xhat == nullptr || xq == nullptr || xs == nullptr) return fail(SERQ_EINVAL, "NULL pointer");
    if (r > 0 && (xsq == nullptr || xss == nullptr)) return fail(SERQ_EINVAL, "r > 0 needs xsq and xss");
    if (!aligned16(Xhat) || !aligned16(xq) || !aligned16(xs) || (r > 0 && (!aligned16(xsq) || !aligned16(xss))))
        return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int rp = residual_width(r);
    const uint4* X = static_cast<const uint4*>(Xhat);
    if (fmt == SERQ_FMT_INT4) {
        if (K <= 16384)
            quant_act_int4_kernel<8><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, static_cast<uint32_t*>(xq),
                                                                  static_cast<float*>(xs),
                                                                  static_cast<uint32_t*>(xsq),
                                                                  static_cast<float*>(xss));
        else
            quant_act_int4_kernel<16><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, static_cast<uint32_t*>(xq),
                                                                   static_cast<float*>(xs),
                                                                   static_cast<uint32_t*>(xsq),
                                                                   static_cast<float*>(xss));
    } else {
        quant_act_mxfp4_kernel<<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, static_cast<uint32_t*>(xq),
                                                            static_cast<uint8_t*>(xs), static_cast<uint32_t*>(xsq),
                                                            static_cast<uint8_t*>(xss));
    }
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

serq_status serq_linear(const serq_weight* w, int M, const void* xq, const void* xs, const void* xsq,
                        const void* xss, void* Y, int32_t* acc_dbg, serq_stream stream) {
    if (w == nullptr) return fail(SERQ_EINVAL, "weight is NULL");
    if (M < 1) return fail(SERQ_EINVAL, "M must be >= 1");
    if (xq == nullptr || xs == nullptr || Y == nullptr) return fail(SERQ_EINVAL, "NULL pointer");
    if (w->rp > 0 && (xsq == nullptr || xss == nullptr)) return fail(SERQ_EINVAL, "r > 0 needs xsq and xss");
    if (!aligned16(xq) || !aligned16(xs) || !aligned16(Y) || (w->rp > 0 && (!aligned16(xsq) || !aligned16(xss))) ||
        !aligned16(acc_dbg))
        return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    if (acc_dbg != nullptr && w->fmt != SERQ_FMT_INT4) return fail(SERQ_EINVAL, "acc_dbg is INT4-only");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    if (dev != w->device) return fail(SERQ_EINVAL, "weight lives on device %d, current device is %d", w->device, dev);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    const int K = w->K, N = w->N, rp = w->rp;
    if (w->fmt == SERQ_FMT_MXFP4 && M <= kMaxDecodeTokens) {
        const int n_tok = M <= 8 ? 8 : 16;
        CUtensorMap tm_x, tm_xr;
        if (serq_status st = make_map(&tm_x, xq, K / 2, M, 128, n_tok, true)) return st;
        if (rp > 0) {
            if (serq_status st = make_map(&tm_xr, xsq, rp / 2, M, 128, n_tok, true)) return st;
        } else {
            tm_xr = tm_x;
        }
        if (serq_status st = decode_setup(info)) return st;
        MxDecodeParams p;
        p.M = M;
        p.N = N;
        p.K = K;
        p.rp = rp;
        p.n_tokens_mma = n_tok;
        p.k_tiles_main = (K + mxd::BK - 1) / mxd::BK;
        p.k_tiles_total = p.k_tiles_main + (rp + mxd::BK - 1) / mxd::BK;
        const int n_blocks = N / mxd::BM;
        p.splits = decode_splits(n_blocks, p.k_tiles_total, info->sms);
        p.atoms_k_main = K / 128;
        p.atoms_k_res = (rp + 127) / 128;
        p.sf_w = static_cast<const uint8_t*>(w->wsc);
        p.sf_x = static_cast<const uint8_t*>(xs);
        p.sf_wr = static_cast<const uint8_t*>(w->rsc);
        p.sf_xr = static_cast<const uint8_t*>(xss);
        p.partial = nullptr;  // cluster form: partial sums stay in shared memory
        p.tickets = nullptr;
        p.Y = static_cast<__nv_bfloat16*>(Y);
        // the S splits of an output block form one cluster; programmatic dependent
        // launch lets the weight stream start under the preceding kernel's tail
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(n_blocks, p.splits, 1);
        cfg.blockDim = dim3(mxd::THREADS, 1, 1);
        cfg.dynamicSmemBytes = mxd::SMEM_BYTES;
        cfg.stream = cs;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = static_cast<unsigned>(p.splits);
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        SERQ_CUDA(cudaLaunchKernelEx(&cfg, serq_linear_mxfp4_decode_kernel<true>, w->tm_w128, tm_x, w->tm_r128, tm_xr,
                                     p));
        return SERQ_OK;
    }

    const uint32_t bi = box_inner_bytes(w->fmt);
    const bool swz = w->fmt == SERQ_FMT_MXFP4;
    CUtensorMap tm_a, tm_ar;
    if (serq_status st = make_map(&tm_a, xq, K / 2, M, bi, 128, swz)) return st;
    if (rp > 0) {
        if (serq_status st = make_map(&tm_ar, xsq, rp / 2, M, bi, 128, swz)) return st;
    } else {
        tm_ar = tm_a;
    }
    const int num_m = (M + 127) / 128;
    const int num_n = (N + 255) / 256;
    const int tiles = num_m * num_n;
    const int grid = tiles < info->sms ? tiles : info->sms;

    if (w->fmt == SERQ_FMT_MXFP4 && M > 128) {
        // CTA-pair kernel: 256 x 256 tiles, B halves split across the pair
        if (!info->smem_set_mxp) {
            SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           mxp::SMEM_BYTES));
            cudaLaunchConfig_t qc = {};
            qc.gridDim = dim3(info->sms, 1, 1);
            qc.blockDim = dim3(mxp::THREADS, 1, 1);
            qc.dynamicSmemBytes = mxp::SMEM_BYTES;
            cudaLaunchAttribute attr;
            attr.id = cudaLaunchAttributeClusterDimension;
            attr.val.clusterDim.x = 2;
            attr.val.clusterDim.y = 1;
            attr.val.clusterDim.z = 1;
            qc.attrs = &attr;
            qc.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, serq_linear_mxfp4_pair_kernel, &qc) != cudaSuccess || n < 1) {
                cudaGetLastError();
                n = info->sms / 2;
            }
            info->pair_clusters = n;
            info->smem_set_mxp = true;
        }
        CUtensorMap tm_b128, tm_br128;
        tm_b128 = w->tm_w128;
        tm_br128 = w->tm_r128;
        MxPairParams p;
        p.M = M;
        p.N = N;
        p.K = K;
        p.rp = rp;
        p.num_n_tiles = (N + mxp::BN - 1) / mxp::BN;
        p.num_m_pairs = (M + 2 * mxp::BM - 1) / (2 * mxp::BM);
        p.num_tiles = p.num_n_tiles * p.num_m_pairs;
        p.k_tiles_main = (K + mxp::BK - 1) / mxp::BK;
        p.k_tiles_res = (rp + mxp::BK - 1) / mxp::BK;
        p.atoms_k_main = K / 128;
        p.atoms_k_res = (rp + 127) / 128;
        p.Y = static_cast<__nv_bfloat16*>(Y);
        const size_t row_blocks_a = static_cast<size_t>((M + 127) / 128);
        MxPairScaleMaps sf;
        if (serq_status st = make_scale_map(&sf.sfa, xs, row_blocks_a * p.atoms_k_main * 512)) return st;
        sf.sfb = w->tm_wsf;
        if (rp > 0) {
            if (serq_status st = make_scale_map(&sf.sfa_r, xss, row_blocks_a * p.atoms_k_res * 512)) return st;
        } else {
            sf.sfa_r = sf.sfa;
        }
        sf.sfb_r = w->tm_rsf;
        const int pairs = info->pair_clusters;
        const int grid2 = 2 * (p.num_tiles < pairs ? p.num_tiles : pairs);
        serq_linear_mxfp4_pair_kernel<<<grid2, mxp::THREADS, mxp::SMEM_BYTES, cs>>>(tm_a, tm_b128, tm_ar, tm_br128,
                                                                                    sf, p);
    } else if (w->fmt == SERQ_FMT_MXFP4) {
        if (!info->smem_set_mx) {
            SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           mx::SMEM_BYTES));
            info->smem_set_mx = true;
        }
        MxParams p;
        p.M = M;
        p.N = N;
        p.K = K;
        p.rp = rp;
        p.num_m_tiles = num_m;
        p.num_tiles = tiles;
        p.k_tiles_main = (K + mx::BK - 1) / mx::BK;
        p.k_tiles_res = (rp + mx::BK - 1) / mx::BK;
        p.atoms_k_main = K / 128;
        p.atoms_k_res = (rp + 127) / 128;
        p.sfa = static_cast<const uint8_t*>(xs);
        p.sfb = static_cast<const uint8_t*>(w->wsc);
        p.sfa_r = static_cast<const uint8_t*>(xss);
        p.sfb_r = static_cast<const uint8_t*>(w->rsc);
        p.Y = static_cast<__nv_bfloat16*>(Y);
        serq_linear_mxfp4_kernel<<<grid, mx::THREADS, mx::SMEM_BYTES, cs>>>(tm_a, w->tm_w, tm_ar, w->tm_r, p);
    } else {
        if (!info->smem_set_i4) {
            SERQ_CUDA(cudaFuncSetAttribute(serq_linear_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           i4::SMEM_BYTES));
            info->smem_set_i4 = true;
        }
        I4Params p;
        p.M = M;
        p.N = N;
        p.K = K;
        p.rp = rp;
        p.num_m_tiles = num_m;
        p.num_tiles = tiles;
        p.k_tiles_main = K / i4::BK;
        p.k_tiles_res = (rp + i4::BK - 1) / i4::BK;
        p.sx = static_cast<const float*>(xs);
        p.sxs = static_cast<const float*>(xss);
        p.sw = static_cast<const float*>(w->wsc);
        p.sR = static_cast<const float*>(w->rsc);
        p.Y = static_cast<__nv_bfloat16*>(Y);
        p.acc_dbg = acc_dbg;
        serq_linear_int4_kernel<<<grid, i4::THREADS, i4::SMEM_BYTES, cs>>>(tm_a, w->tm_w, tm_ar, w->tm_r, p);
    }
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

serq_status serq_linear_small_m_noalloc(int M, int K, int N, int r, const void* wq, const void* w_scale,
                                        const void* rq, const void* r_scale, const void* xq, const void* xs,
                                        const void* xsq, const void* xss, void* Y, serq_stream stream) {
    if (M < 1 || M > kMaxDecodeTokens) return fail(SERQ_EINVAL, "M=%d outside 1..%d", M, kMaxDecodeTokens);
    if (K < 128 || K % 128 != 0 || K > 32768 || N < 128 || N % 128 != 0 || r < 0 || r > K)
        return fail(SERQ_EINVAL, "bad shape K=%d N=%d r=%d (need K%%128==0, K<=32768, N%%128==0, 0<=r<=K)", K, N, r);
    if (static_cast<size_t>(N / 128) * 4u > kNoAllocTicketBytes)
        return fail(SERQ_EINVAL, "N=%d above the static scratch limit of %zu output channels", N,
                    kNoAllocTicketBytes / 4u * 128u);
    const size_t cap_floats = (kNoAllocScratchBytes - kNoAllocTicketBytes) / sizeof(float);
    if (static_cast<size_t>(M) * N > cap_floats)
        return fail(SERQ_EINVAL, "M*N=%zu above the static scratch limit of %zu", static_cast<size_t>(M) * N,
                    cap_floats);
    const int rp = residual_width(r);
    if (wq == nullptr || w_scale == nullptr || xq == nullptr || xs == nullptr || Y == nullptr)
        return fail(SERQ_EINVAL, "NULL pointer");
    if (rp > 0 && (rq == nullptr || r_scale == nullptr || xsq == nullptr || xss == nullptr))
        return fail(SERQ_EINVAL, "r > 0 needs rq, r_scale, xsq and xss");
    if (!aligned16(wq) || !aligned16(w_scale) || !aligned16(xq) || !aligned16(xs) || !aligned16(Y) ||
        (rp > 0 && (!aligned16(rq) || !aligned16(r_scale) || !aligned16(xsq) || !aligned16(xss))))
        return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    void* scratch = nullptr;
    if (serq_status st = noalloc_scratch(dev, &scratch)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    const int n_tok = M <= 8 ? 8 : 16;
    CUtensorMap tm_w, tm_wr, tm_x, tm_xr;
    if (serq_status st = make_map(&tm_w, wq, K / 2, N, 128, 128, true)) return st;
    if (serq_status st = make_map(&tm_x, xq, K / 2, M, 128, n_tok, true)) return st;
    if (rp > 0) {
        if (serq_status st = make_map(&tm_wr, rq, rp / 2, N, 128, 128, true)) return st;
        if (serq_status st = make_map(&tm_xr, xsq, rp / 2, M, 128, n_tok, true)) return st;
    } else {
        tm_wr = tm_w;
        tm_xr = tm_x;
    }
    if (serq_status st = decode_setup(info)) return st;
    MxDecodeParams p;
    p.M = M;
    p.N = N;
    p.K = K;
    p.rp = rp;
    p.n_tokens_mma = n_tok;
    p.k_tiles_main = (K + mxd::BK - 1) / mxd::BK;
    p.k_tiles_total = p.k_tiles_main + (rp + mxd::BK - 1) / mxd::BK;
    const int n_blocks = N / mxd::BM;
    int splits = decode_splits(n_blocks, p.k_tiles_total, info->sms);
    while (splits > 1 && static_cast<size_t>(splits) * M * N > cap_floats) --splits;
    p.splits = splits;
    p.atoms_k_main = K / 128;
    p.atoms_k_res = (rp + 127) / 128;
    p.sf_w = static_cast<const uint8_t*>(w_scale);
    p.sf_x = static_cast<const uint8_t*>(xs);
    p.sf_wr = static_cast<const uint8_t*>(r_scale);
    p.sf_xr = static_cast<const uint8_t*>(xss);
    p.tickets = static_cast<unsigned int*>(scratch);
    p.partial = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kNoAllocTicketBytes);
    p.Y = static_cast<__nv_bfloat16*>(Y);
    // the array keeps the previous call's contents: the tickets must start at zero
    SERQ_CUDA(cudaMemsetAsync(p.tickets, 0, static_cast<size_t>(n_blocks) * sizeof(unsigned int), cs));
    serq_linear_mxfp4_decode_kernel<false><<<dim3(n_blocks, splits), mxd::THREADS, mxd::SMEM_BYTES, cs>>>(
        tm_w, tm_x, tm_wr, tm_xr, p);
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

serq_status serq_selftest_wait(long long limit_cycles, int arrive, serq_stream stream) {
    if (limit_cycles < 1 || limit_cycles > 4000000000LL)
        return fail(SERQ_EINVAL, "limit_cycles=%lld outside 1..4e9", limit_cycles);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    wait_selftest_kernel<<<1, 32, 0, cs>>>(limit_cycles, arrive != 0 ? 1 : 0);
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

serq_status serq_device_status(serq_stream stream) {
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    SERQ_CUDA(cudaStreamSynchronize(cs));
    unsigned int flag = 0;
    SERQ_CUDA(cudaMemcpyFromSymbol(&flag, g_timeout_flag, sizeof(flag)));
    if (flag != 0) {
        const unsigned int zero = 0;
        SERQ_CUDA(cudaMemcpyToSymbol(g_timeout_flag, &zero, sizeof(zero)));
        return fail(SERQ_ETIMEOUT, "a kernel pipeline wait timed out (site 0x%x)", flag);
    }
    return SERQ_OK;
}

}  // extern "C"
