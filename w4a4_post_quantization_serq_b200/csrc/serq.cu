// C ABI of the SERQ W4A4 linear (include/serq.h): argument checks, device
// buffers of prepared weights, tensor-map encoding and kernel launches.
// The kernels themselves live in the *.cuh files of this directory; this is
// the only translation unit, so they share one device-side timeout flag.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "serq.h"

#include "ptx.cuh"
#include "quant_act.cuh"
#include "producer.cuh"
#include "block.cuh"
#include "attention_tc.cuh"
#include "prepare.cuh"
#include "gemm_mxfp4.cuh"
#include "gemm_int4.cuh"
#include "gemm_mxfp4_decode.cuh"
#include "gemm_mxfp4_pair.cuh"
#include "weight_format.h"

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

// INT4 weights (per-output-channel fp32 scales): the W4A4 and W4A8 formats.
bool int_weights(int fmt) { return fmt == SERQ_FMT_INT4 || fmt == SERQ_FMT_W4A8; }

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
    bool smem_set_prod = false;
    int pair_clusters = 0;  // co-resident 2-CTA clusters of the pair kernel
    cudaMemPool_t scratch_pool = nullptr;  // stream-ordered scratch that is kept once grown
};

// split-K ranges of the small-M kernel. Two CTAs fit per SM. A launch first
// takes one CTA per SM, leaving the other slot to the next launch, whose CTAs
// then prefetch their weight stages while this one finishes; when a CTA
// would still have more than one K-tile beyond what its ring holds, the
// launch takes both slots instead (more bytes in flight; one refill per CTA
// costs less than giving up that overlap: 4096 x 6144 runs 6.9 us with 144
// CTAs against 10.1 us with 288). At most kMaxDecodeSplits (the
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
    return (k_tiles + s1 - 1) / s1 > mxd::STAGES + 1 ? fit(2 * sms) : s1;
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

// The library's stream-ordered scratch pool of a device (created on first use):
// memory freed into it stays reserved for the next allocation instead of
// going back to the driver at each synchronization. The process's default
// pool is left as it is.
serq_status scratch_pool(int dev, DeviceInfo* info, cudaMemPool_t* out) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (info->scratch_pool == nullptr) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        SERQ_CUDA(cudaMemPoolCreate(&pool, &props));
        uint64_t keep = ~uint64_t(0);
        SERQ_CUDA(cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep));
        info->scratch_pool = pool;
    }
    *out = info->scratch_pool;
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

// MXFP4 activation scale atoms (`bytes`, a multiple of 512) as the 3-D view
// the CTA-pair kernel reads its wide scale tiles through: x = byte within a
// 128-byte piece, y = atom (stride 512), z = piece of the atom (stride 128);
// a box of 128 x 2 x 4 is a K-tile's two atoms, pieces outermost.
serq_status make_sfa_wide_map(CUtensorMap* map, const void* base, size_t bytes) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return fail(SERQ_ECUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[3] = {128, bytes / 512, 4};
    const cuuint64_t strides[2] = {512, 128};
    const cuuint32_t box[3] = {128, 2, 4};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SERQ_ECUDA, "cuTensorMapEncodeTiled (scale view) failed (%d)", static_cast<int>(r));
    return SERQ_OK;
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
    float* tmp_b;          // preparation scratch at the end of the arena
    unsigned int* tmp_col;
    // gate/up weight with the SwiGLU producer of a down linear folded in
    // (serq_prepare_swiglu): its own allocation of down's 1/s[perm], F floats
    float* swiglu_inv_s;
    int swiglu_F, swiglu_r, swiglu_rp;
};

namespace {

// Test hook: the next n device allocations of a weight fail with SERQ_ENOMEM
// without calling cudaMalloc (serq_debug_fail_next_allocations).
std::atomic<int> g_fail_allocs{0};

serq_status check_weight_shape(int K, int N, int r, int fmt) {
    if (K < 128 || K % 128 != 0 || K > 32768 || N < 128 || N % 128 != 0 || r < 0 || r > K)
        return fail(SERQ_EINVAL, "bad shape K=%d N=%d r=%d (need K%%128==0, K<=32768, N%%128==0, 0<=r<=K)", K, N, r);
    if (fmt != SERQ_FMT_INT4 && fmt != SERQ_FMT_MXFP4 && fmt != SERQ_FMT_W4A8) return fail(SERQ_EINVAL, "unknown format %d", fmt);
    return SERQ_OK;
}

// One device arena per weight: perm, s, s_perm, inv_s, W^_q and its scales,
// Q(R) and its scales, the wide MXFP4 scale copies, then preparation scratch.
// Zero-filled on `cs`. Nothing is left allocated on failure.
serq_status weight_alloc(int K, int N, int r, int fmt, int dev, cudaStream_t cs, serq_weight** out) {
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
    if (int_weights(fmt)) {
        w->wsc_bytes = static_cast<size_t>(N) * 4;
        w->rsc_bytes = static_cast<size_t>(N) * 4;
    } else {
        w->wsc_bytes = atom_bytes(N, K / 32);
        w->rsc_bytes = rp > 0 ? atom_bytes(N, rp / 32) : 0;
        const size_t pairs = static_cast<size_t>((N / 128 + 1) / 2);
        w->wscw_bytes = pairs * (K / 128) * 4096;
        w->rscw_bytes = rp > 0 ? pairs * ((rp + 127) / 128) * 4096 : 0;
    }
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
    const size_t o_b = take(4u * K), o_col = take(4u * N);
    int pending = g_fail_allocs.load();
    while (pending > 0 && !g_fail_allocs.compare_exchange_weak(pending, pending - 1)) {
    }
    if (pending > 0) {
        delete w;
        return fail(SERQ_ENOMEM, "device allocation of %zu bytes failed (injected by the test hook)", off);
    }
    void* arena = nullptr;
    const cudaError_t ae = cudaMalloc(&arena, off);
    if (ae != cudaSuccess) {
        delete w;
        cudaGetLastError();
        return fail(SERQ_ENOMEM, "cudaMalloc(%zu) failed: %s", off, cudaGetErrorString(ae));
    }
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
    w->tmp_b = reinterpret_cast<float*>(base + o_b);
    w->tmp_col = reinterpret_cast<unsigned int*>(base + o_col);
    const cudaError_t me = cudaMemsetAsync(arena, 0, off, cs);
    if (me != cudaSuccess) {
        cudaFree(arena);
        delete w;
        return cuda_fail(me, "cudaMemsetAsync(weight arena)");
    }
    *out = w;
    return SERQ_OK;
}

// After the packed tensors are in place: the wide MXFP4 scale copies of the
// CTA-pair kernel, then the tensor maps. Synchronizes `cs`.
serq_status weight_finish(serq_weight* w, cudaStream_t cs) {
    const int K = w->K, N = w->N, rp = w->rp, fmt = w->fmt;
    if (fmt == SERQ_FMT_MXFP4) {
        scale_widen_kernel<<<static_cast<unsigned>((w->wscw_bytes / 16 + 255) / 256), 256, 0, cs>>>(
            static_cast<const uint8_t*>(w->wsc), N / 128, K / 128, w->wscw, w->wscw_bytes);
        if (rp > 0)
            scale_widen_kernel<<<static_cast<unsigned>((w->rscw_bytes / 16 + 255) / 256), 256, 0, cs>>>(
                static_cast<const uint8_t*>(w->rsc), N / 128, (rp + 127) / 128, w->rscw, w->rscw_bytes);
        SERQ_CUDA(cudaGetLastError());
    }
    SERQ_CUDA(cudaStreamSynchronize(cs));
    const uint32_t bi = box_inner_bytes(fmt);
    const bool swz = fmt == SERQ_FMT_MXFP4;
    if (serq_status st = make_map(&w->tm_w, w->wq, K / 2, N, bi, 256, swz)) return st;
    if (rp > 0) {
        if (serq_status st = make_map(&w->tm_r, w->rq, rp / 2, N, bi, 256, swz)) return st;
    } else {
        w->tm_r = w->tm_w;
    }
    if (fmt == SERQ_FMT_MXFP4) {
        if (serq_status st = make_map(&w->tm_w128, w->wq, K / 2, N, 128, 128, true)) return st;
        if (serq_status st = make_map(&w->tm_wsf, w->wscw, 256, w->wscw_bytes / 256, 256, 32, false)) return st;
        if (rp > 0) {
            if (serq_status st = make_map(&w->tm_rsf, w->rscw, 256, w->rscw_bytes / 256, 256, 32, false)) return st;
            if (serq_status st = make_map(&w->tm_r128, w->rq, rp / 2, N, 128, 128, true)) return st;
        } else {
            w->tm_rsf = w->tm_wsf;
            w->tm_r128 = w->tm_w128;
        }
    }
    return SERQ_OK;
}

}  // namespace

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
    if (fmt != SERQ_FMT_INT4 && fmt != SERQ_FMT_MXFP4 && fmt != SERQ_FMT_W4A8) return fail(SERQ_EINVAL, "unknown format %d", fmt);
    const int rp = residual_width(r);
    out->xq = static_cast<size_t>(M) * (K / 2);
    out->xsq = static_cast<size_t>(M) * (rp / 2);
    if (fmt == SERQ_FMT_W4A8) {  // one int8 code per element
        out->xq = static_cast<size_t>(M) * K;
        out->xsq = static_cast<size_t>(M) * rp;
    }
    if (int_weights(fmt)) {
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
    if (w->arena != nullptr || w->swiglu_inv_s != nullptr) {
        int cur = -1;
        cudaGetDevice(&cur);
        if (cur != w->device) cudaSetDevice(w->device);
        if (w->arena != nullptr) cudaFree(w->arena);
        if (w->swiglu_inv_s != nullptr) cudaFree(w->swiglu_inv_s);
        if (cur != w->device && cur >= 0) cudaSetDevice(cur);
    }
    delete w;
}

serq_status serq_prepare(const serq_prepare_desc* desc, serq_weight** out, serq_stream stream) {
    if (desc == nullptr || out == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    *out = nullptr;
    const int K = desc->K, N = desc->N, r = desc->r, fmt = desc->fmt;
    if (serq_status st = check_weight_shape(K, N, r, fmt)) return st;
    if (desc->W == nullptr || !aligned16(desc->W)) return fail(SERQ_EINVAL, "W must be a 16-byte aligned pointer");
    if ((desc->act_absmax == nullptr) == (desc->s == nullptr))
        return fail(SERQ_EINVAL, "give exactly one of act_absmax and s");
    if (desc->R != nullptr && (!aligned16(desc->R) || r < 1))
        return fail(SERQ_EINVAL, "a given residual needs r >= 1 and a 16-byte aligned pointer");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    serq_weight* w = nullptr;
    if (serq_status st = weight_alloc(K, N, r, fmt, dev, cs, &w)) return st;
    const int rp = w->rp;
    float* tmp_b = w->tmp_b;
    unsigned int* tmp_col = w->tmp_col;

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
    const __nv_bfloat16* G = static_cast<const __nv_bfloat16*>(desc->R);  // given residual, or NULL
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
    if (int_weights(fmt)) {
        const int rows = 128;
        weight_colamax_kernel<<<dim3(N / 256 + (N % 256 != 0), (K + rows - 1) / rows), 256, 0, cs>>>(W, w->s, K, N,
                                                                                                    rows, tmp_col);
        weight_quant_int4_kernel<<<qgrid, qblock, 0, cs>>>(W, w->perm, w->s_perm, tmp_col, K, N, w->wq,
                                                           static_cast<float*>(w->wsc));
        if (r > 0 && G != nullptr)
            given_residual_int4_kernel<<<(N + 127) / 128, 128, 0, cs>>>(G, N, r, rp, w->rq, static_cast<float*>(w->rsc));
        else if (r > 0)
            residual_int4_kernel<<<(N + 127) / 128, 128, 0, cs>>>(W, w->perm, w->s_perm,
                                                                  static_cast<const float*>(w->wsc), N, r, rp, w->rq,
                                                                  static_cast<float*>(w->rsc));
    } else {
        weight_quant_mxfp4_kernel<<<qgrid, qblock, 0, cs>>>(W, w->perm, w->s_perm, K, N, w->wq,
                                                            static_cast<uint8_t*>(w->wsc));
        if (r > 0 && G != nullptr)
            given_residual_mxfp4_kernel<<<dim3(N / 32, (rp / 32 + 7) / 8), qblock, 0, cs>>>(
                G, N, r, rp, w->rq, static_cast<uint8_t*>(w->rsc));
        else if (r > 0)
            residual_mxfp4_kernel<<<dim3(N / 32, (rp / 32 + 7) / 8), qblock, 0, cs>>>(
                W, w->perm, w->s_perm, K, N, r, rp, w->rq, static_cast<uint8_t*>(w->rsc));
    }
    PREP_CUDA(cudaGetLastError());
    if (serq_status st = weight_finish(w, cs)) return bail(st);
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

}  // extern "C"

// ============================================================== checkpoint / export / import
namespace {

bool is_int4_code_ok(uint8_t nib) { return (nib & 0xF) != 0x8; }  // -8 never occurs

// Checks the canonical host form (see serq_weight_host in serq.h).
serq_status check_host_weight(const serq_weight_host* h) {
    if (serq_status st = check_weight_shape(h->K, h->N, h->r, h->fmt)) return st;
    const int K = h->K, N = h->N, r = h->r, rp = h->rp, fmt = h->fmt;
    if (rp != residual_width(r)) return fail(SERQ_EINVAL, "rp=%d, expected round_up(r, 64) = %d", rp, residual_width(r));
    if (h->perm == nullptr || h->s == nullptr || h->inv_s == nullptr || h->wq == nullptr || h->w_scale == nullptr)
        return fail(SERQ_EINVAL, "NULL part (perm, s, inv_s, wq and w_scale are required)");
    if (rp > 0 && (h->rq == nullptr || h->r_scale == nullptr)) return fail(SERQ_EINVAL, "r > 0 needs rq and r_scale");
    std::vector<uint8_t> seen(static_cast<size_t>(K), 0);
    for (int i = 0; i < K; ++i) {
        const int j = h->perm[i];
        if (j < 0 || j >= K || seen[j]) return fail(SERQ_EINVAL, "perm is not a permutation of 0..K-1 (at %d)", i);
        seen[j] = 1;
    }
    for (int j = 0; j < K; ++j)
        if (!std::isfinite(h->s[j]) || !(h->s[j] > 0.0f)) return fail(SERQ_EINVAL, "s[%d] is not finite and > 0", j);
    for (int i = 0; i < K; ++i) {
        const float want = 1.0f / h->s[h->perm[i]];
        if (std::memcmp(&want, &h->inv_s[i], 4) != 0) return fail(SERQ_EINVAL, "inv_s[%d] != 1/s[perm[%d]]", i, i);
    }
    const size_t wq_bytes = static_cast<size_t>(N) * (K / 2);
    const size_t rq_row = static_cast<size_t>(rp / 2);
    if (int_weights(fmt)) {
        for (size_t i = 0; i < wq_bytes; ++i)
            if (!is_int4_code_ok(h->wq[i]) || !is_int4_code_ok(h->wq[i] >> 4))
                return fail(SERQ_EINVAL, "INT4 code -8 in wq (byte %zu)", i);
        const float* ws = static_cast<const float*>(h->w_scale);
        for (int n = 0; n < N; ++n)
            if (!std::isfinite(ws[n]) || ws[n] < 0.0f) return fail(SERQ_EINVAL, "w_scale[%d] not finite >= 0", n);
        if (h->r_scale != nullptr) {
            const float* rs = static_cast<const float*>(h->r_scale);
            for (int n = 0; n < N; ++n)
                if (!std::isfinite(rs[n]) || rs[n] < 0.0f || (rp == 0 && rs[n] != 0.0f))
                    return fail(SERQ_EINVAL, "r_scale[%d] not finite >= 0 (or nonzero with r = 0)", n);
        }
    } else {
        const uint8_t* ws = static_cast<const uint8_t*>(h->w_scale);
        for (size_t i = 0; i < static_cast<size_t>(N) * (K / 32); ++i)
            if (ws[i] == 0xFF) return fail(SERQ_EINVAL, "E8M0 byte 0xFF in w_scale");
        if (rp > 0) {
            const uint8_t* rs = static_cast<const uint8_t*>(h->r_scale);
            const int nbr = rp / 32, used = (r + 31) / 32;
            for (int n = 0; n < N; ++n)
                for (int b = 0; b < nbr; ++b) {
                    const uint8_t e = rs[static_cast<size_t>(n) * nbr + b];
                    if (e == 0xFF || (b >= used && e != 0))
                        return fail(SERQ_EINVAL, "r_scale row %d block %d: 0xFF or nonzero past r", n, b);
                }
        }
    }
    for (int n = 0; n < N && rp > 0; ++n)
        for (int c = r; c < rp; ++c) {
            const uint8_t byte = h->rq[static_cast<size_t>(n) * rq_row + c / 2];
            const uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 0xF);
            if (nib != 0) return fail(SERQ_EINVAL, "rq row %d: nonzero code at position %d >= r", n, c);
        }
    if (int_weights(fmt) && rp > 0)
        for (size_t i = 0; i < static_cast<size_t>(N) * rq_row; ++i)
            if (!is_int4_code_ok(h->rq[i]) || !is_int4_code_ok(h->rq[i] >> 4))
                return fail(SERQ_EINVAL, "INT4 code -8 in rq (byte %zu)", i);
    return SERQ_OK;
}

// Owning host copy of the canonical parts.
struct HostWeight {
    serq_weight_host h{};
    std::vector<uint8_t> buf;
    void allocate(int fmt, int K, int N, int r, int rp) {
        const wfmt::Sizes z = wfmt::canonical_sizes(fmt, K, N, rp);
        buf.assign(z.total(), 0);
        uint8_t* p = buf.data();
        h.K = K;
        h.N = N;
        h.r = r;
        h.rp = rp;
        h.fmt = fmt;
        h.perm = reinterpret_cast<int32_t*>(p);
        p += z.perm;
        h.s = reinterpret_cast<float*>(p);
        p += z.s;
        h.inv_s = reinterpret_cast<float*>(p);
        p += z.inv_s;
        h.wq = p;
        p += z.wq;
        h.w_scale = p;
        p += z.w_scale;
        h.rq = z.rq > 0 ? p : nullptr;
        p += z.rq;
        h.r_scale = z.r_scale > 0 ? p : nullptr;
    }
};

struct FileCloser {
    FILE* f;
    ~FileCloser() {
        if (f != nullptr) fclose(f);
    }
};

serq_status write_file(const char* path, const serq_weight_host* h) {
    const wfmt::Sizes z = wfmt::canonical_sizes(h->fmt, h->K, h->N, h->rp);
    const void* parts[7] = {h->perm, h->s, h->inv_s, h->wq, h->w_scale, h->rq, h->r_scale};
    const size_t sizes[7] = {z.perm, z.s, z.inv_s, z.wq, z.w_scale, z.rq, z.r_scale};
    std::vector<uint8_t> zeros;
    wfmt::Header hd;
    std::memset(&hd, 0, sizeof(hd));
    std::memcpy(hd.magic, wfmt::kMagic, 8);
    hd.version = wfmt::kVersion;
    hd.fmt = h->fmt;
    hd.K = h->K;
    hd.N = h->N;
    hd.r = h->r;
    hd.rp = h->rp;
    hd.payload_bytes = z.total();
    uint64_t ck = 1469598103934665603ull;
    for (int i = 0; i < 7; ++i) {
        if (sizes[i] == 0) continue;
        const uint8_t* src = static_cast<const uint8_t*>(parts[i]);
        if (src == nullptr) {  // only r_scale of INT4 with r = 0 may be absent: zeros
            zeros.assign(sizes[i], 0);
            src = zeros.data();
        }
        ck = wfmt::fnv1a64(src, sizes[i], ck);
    }
    hd.checksum = ck;
    FileCloser fc{fopen(path, "wb")};
    if (fc.f == nullptr) return fail(SERQ_EINVAL, "cannot open %s for writing", path);
    if (fwrite(&hd, sizeof(hd), 1, fc.f) != 1) return fail(SERQ_EINVAL, "write to %s failed", path);
    for (int i = 0; i < 7; ++i) {
        if (sizes[i] == 0) continue;
        const void* src = parts[i];
        if (src == nullptr) {
            zeros.assign(sizes[i], 0);
            src = zeros.data();
        }
        if (fwrite(src, 1, sizes[i], fc.f) != sizes[i]) return fail(SERQ_EINVAL, "write to %s failed", path);
    }
    if (fclose(fc.f) != 0) {
        fc.f = nullptr;
        return fail(SERQ_EINVAL, "closing %s failed", path);
    }
    fc.f = nullptr;
    return SERQ_OK;
}

// Reads and checks a checkpoint into an owning host copy.
serq_status read_file(const char* path, HostWeight* hw) {
    FileCloser fc{fopen(path, "rb")};
    if (fc.f == nullptr) return fail(SERQ_EINVAL, "cannot open %s", path);
    wfmt::Header hd;
    if (fread(&hd, sizeof(hd), 1, fc.f) != 1) return fail(SERQ_EINVAL, "%s: truncated header", path);
    if (std::memcmp(hd.magic, wfmt::kMagic, 8) != 0) return fail(SERQ_EINVAL, "%s: not a SERQ weight file", path);
    if (hd.version != wfmt::kVersion) return fail(SERQ_EINVAL, "%s: unsupported version %u", path, hd.version);
    if (serq_status st = check_weight_shape(hd.K, hd.N, hd.r, hd.fmt)) return st;
    if (hd.rp != residual_width(hd.r)) return fail(SERQ_EINVAL, "%s: inconsistent rp", path);
    const wfmt::Sizes z = wfmt::canonical_sizes(hd.fmt, hd.K, hd.N, hd.rp);
    if (hd.payload_bytes != z.total()) return fail(SERQ_EINVAL, "%s: payload size mismatch", path);
    hw->allocate(hd.fmt, hd.K, hd.N, hd.r, hd.rp);
    if (fread(hw->buf.data(), 1, hw->buf.size(), fc.f) != hw->buf.size())
        return fail(SERQ_EINVAL, "%s: truncated payload", path);
    if (fgetc(fc.f) != EOF) return fail(SERQ_EINVAL, "%s: trailing bytes after the payload", path);
    if (wfmt::fnv1a64(hw->buf.data(), hw->buf.size()) != hd.checksum) return fail(SERQ_EINVAL, "%s: checksum mismatch", path);
    return check_host_weight(&hw->h);
}

serq_status copy_parts(const serq_weight_host* src, serq_weight_host* dst) {
    const wfmt::Sizes z = wfmt::canonical_sizes(src->fmt, src->K, src->N, src->rp);
    dst->K = src->K;
    dst->N = src->N;
    dst->r = src->r;
    dst->rp = src->rp;
    dst->fmt = src->fmt;
    auto cp = [](void* d, const void* s, size_t n) {
        if (d != nullptr && n > 0) {
            if (s != nullptr)
                std::memcpy(d, s, n);
            else
                std::memset(d, 0, n);
        }
    };
    cp(dst->perm, src->perm, z.perm);
    cp(dst->s, src->s, z.s);
    cp(dst->inv_s, src->inv_s, z.inv_s);
    cp(dst->wq, src->wq, z.wq);
    cp(dst->w_scale, src->w_scale, z.w_scale);
    cp(dst->rq, src->rq, z.rq);
    cp(dst->r_scale, src->r_scale, z.r_scale);
    return SERQ_OK;
}

// Runs `fn` with the weight's device current, restoring the caller's device.
template <class F>
serq_status on_device(int dev, F&& fn) {
    int cur = -1;
    SERQ_CUDA(cudaGetDevice(&cur));
    if (cur != dev) SERQ_CUDA(cudaSetDevice(dev));
    const serq_status st = fn();
    if (cur != dev) cudaSetDevice(cur);
    return st;
}

}  // namespace

extern "C" {

serq_status serq_weight_export(const serq_weight* w, serq_weight_host* dst) {
    if (w == nullptr || dst == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    dst->K = w->K;
    dst->N = w->N;
    dst->r = w->r;
    dst->rp = w->rp;
    dst->fmt = w->fmt;
    return on_device(w->device, [&]() -> serq_status {
        SERQ_CUDA(cudaDeviceSynchronize());
        const int K = w->K, N = w->N, rp = w->rp;
        if (dst->perm != nullptr) SERQ_CUDA(cudaMemcpy(dst->perm, w->perm, 4u * K, cudaMemcpyDeviceToHost));
        if (dst->s != nullptr) SERQ_CUDA(cudaMemcpy(dst->s, w->s, 4u * K, cudaMemcpyDeviceToHost));
        if (dst->inv_s != nullptr) SERQ_CUDA(cudaMemcpy(dst->inv_s, w->inv_s, 4u * K, cudaMemcpyDeviceToHost));
        if (dst->wq != nullptr) SERQ_CUDA(cudaMemcpy(dst->wq, w->wq, w->wq_bytes, cudaMemcpyDeviceToHost));
        if (dst->rq != nullptr && w->rq_bytes > 0)
            SERQ_CUDA(cudaMemcpy(dst->rq, w->rq, w->rq_bytes, cudaMemcpyDeviceToHost));
        if (int_weights(w->fmt)) {
            if (dst->w_scale != nullptr) SERQ_CUDA(cudaMemcpy(dst->w_scale, w->wsc, 4u * N, cudaMemcpyDeviceToHost));
            if (dst->r_scale != nullptr) SERQ_CUDA(cudaMemcpy(dst->r_scale, w->rsc, 4u * N, cudaMemcpyDeviceToHost));
        } else {
            std::vector<uint8_t> atoms;
            if (dst->w_scale != nullptr) {
                atoms.resize(w->wsc_bytes);
                SERQ_CUDA(cudaMemcpy(atoms.data(), w->wsc, w->wsc_bytes, cudaMemcpyDeviceToHost));
                wfmt::atoms_to_rows(atoms.data(), N, K / 32, static_cast<uint8_t*>(dst->w_scale));
            }
            if (dst->r_scale != nullptr && rp > 0) {
                atoms.resize(w->rsc_bytes);
                SERQ_CUDA(cudaMemcpy(atoms.data(), w->rsc, w->rsc_bytes, cudaMemcpyDeviceToHost));
                wfmt::atoms_to_rows(atoms.data(), N, rp / 32, static_cast<uint8_t*>(dst->r_scale));
            }
        }
        return SERQ_OK;
    });
}

serq_status serq_weight_create_from_host(const serq_weight_host* src, serq_weight** out, serq_stream stream) {
    if (src == nullptr || out == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    *out = nullptr;
    if (serq_status st = check_host_weight(src)) return st;
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int K = src->K, N = src->N, rp = src->rp;
    serq_weight* w = nullptr;
    if (serq_status st = weight_alloc(K, N, src->r, src->fmt, dev, cs, &w)) return st;
    auto bail = [&](serq_status st) {
        cudaStreamSynchronize(cs);
        serq_weight_destroy(w);
        return st;
    };
    std::vector<float> s_perm(static_cast<size_t>(K));
    for (int i = 0; i < K; ++i) s_perm[i] = src->s[src->perm[i]];
    std::vector<uint8_t> watoms, ratoms;
    auto up = [&](void* d, const void* h, size_t n) -> serq_status {
        if (n == 0) return SERQ_OK;
        const cudaError_t e = cudaMemcpyAsync(d, h, n, cudaMemcpyHostToDevice, cs);
        return e == cudaSuccess ? SERQ_OK : cuda_fail(e, "cudaMemcpyAsync(weight upload)");
    };
    serq_status st = up(w->perm, src->perm, 4u * K);
    if (!st) st = up(w->s, src->s, 4u * K);
    if (!st) st = up(w->s_perm, s_perm.data(), 4u * K);
    if (!st) st = up(w->inv_s, src->inv_s, 4u * K);
    if (!st) st = up(w->wq, src->wq, w->wq_bytes);
    if (!st && rp > 0) st = up(w->rq, src->rq, w->rq_bytes);
    if (!st) {
        if (int_weights(src->fmt)) {
            st = up(w->wsc, src->w_scale, 4u * N);
            if (!st && src->r_scale != nullptr) st = up(w->rsc, src->r_scale, 4u * N);
        } else {
            watoms.resize(w->wsc_bytes);
            wfmt::rows_to_atoms(static_cast<const uint8_t*>(src->w_scale), N, K / 32, watoms.data());
            st = up(w->wsc, watoms.data(), w->wsc_bytes);
            if (!st && rp > 0) {
                ratoms.resize(w->rsc_bytes);
                wfmt::rows_to_atoms(static_cast<const uint8_t*>(src->r_scale), N, rp / 32, ratoms.data());
                st = up(w->rsc, ratoms.data(), w->rsc_bytes);
            }
        }
    }
    if (!st) st = weight_finish(w, cs);  // synchronizes: the pageable host copies are complete
    if (st) return bail(st);
    *out = w;
    return SERQ_OK;
}

serq_status serq_weight_save(const serq_weight* w, const char* path) {
    if (w == nullptr || path == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    HostWeight hw;
    hw.allocate(w->fmt, w->K, w->N, w->r, w->rp);
    if (serq_status st = serq_weight_export(w, &hw.h)) return st;
    return write_file(path, &hw.h);
}

serq_status serq_weight_load(const char* path, serq_weight** out, serq_stream stream) {
    if (path == nullptr || out == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    *out = nullptr;
    HostWeight hw;
    if (serq_status st = read_file(path, &hw)) return st;
    return serq_weight_create_from_host(&hw.h, out, stream);
}

serq_status serq_weight_file_write(const char* path, const serq_weight_host* src) {
    if (path == nullptr || src == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    if (serq_status st = check_host_weight(src)) return st;
    return write_file(path, src);
}

serq_status serq_weight_file_read(const char* path, serq_weight_host* dst) {
    if (path == nullptr || dst == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    HostWeight hw;
    if (serq_status st = read_file(path, &hw)) return st;
    return copy_parts(&hw.h, dst);
}

int serq_debug_fail_next_allocations(int n) { return g_fail_allocs.exchange(n < 0 ? 0 : n); }

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
    if (fmt != SERQ_FMT_MXFP4) {
        // a CTA per row holding its chunks in registers: the fewest per thread that
        // cover K, so that short rows take few registers and many rows are in flight
        const int per_thread = (K / 8 + kQuantThreads - 1) / kQuantThreads;
        const int maxc = per_thread <= 1 ? 1 : per_thread <= 2 ? 2 : per_thread <= 4 ? 4 : per_thread <= 8 ? 8 : 16;
        float* fxs = static_cast<float*>(xs);
        float* fxss = static_cast<float*>(xss);
        if (fmt == SERQ_FMT_W4A8) {
            auto* q8 = static_cast<uint8_t*>(xq);
            auto* qs8 = static_cast<uint8_t*>(xsq);
            switch (maxc) {
                case 1: quant_act_int8_kernel<1><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q8, fxs, qs8, fxss); break;
                case 2: quant_act_int8_kernel<2><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q8, fxs, qs8, fxss); break;
                case 4: quant_act_int8_kernel<4><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q8, fxs, qs8, fxss); break;
                case 8: quant_act_int8_kernel<8><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q8, fxs, qs8, fxss); break;
                default: quant_act_int8_kernel<16><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q8, fxs, qs8, fxss);
            }
        } else {
            auto* q4 = static_cast<uint32_t*>(xq);
            auto* qs4 = static_cast<uint32_t*>(xsq);
            switch (maxc) {
                case 1: quant_act_int4_kernel<1><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q4, fxs, qs4, fxss); break;
                case 2: quant_act_int4_kernel<2><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q4, fxs, qs4, fxss); break;
                case 4: quant_act_int4_kernel<4><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q4, fxs, qs4, fxss); break;
                case 8: quant_act_int4_kernel<8><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q4, fxs, qs4, fxss); break;
                default: quant_act_int4_kernel<16><<<M, kQuantThreads, 0, cs>>>(X, K, r, rp, q4, fxs, qs4, fxss);
            }
        }
    } else {
        // a CTA per segment of QF_CHUNKS 16-byte chunks of one row
        if (M > 65535) return fail(SERQ_EUNSUPPORTED, "M=%d above 65535", M);
        const dim3 grid((K / 8 + QF_CHUNKS - 1) / QF_CHUNKS, M);
        quant_act_mxfp4_flat_kernel<<<grid, QF_THREADS, 0, cs>>>(
            X, K, r, rp, static_cast<uint32_t*>(xq), static_cast<uint8_t*>(xs), static_cast<uint32_t*>(xsq),
            static_cast<uint8_t*>(xss));
    }
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

}  // extern "C"

namespace {

template <int KIND, int FMT, int MAXC>
serq_status producer_setup_one() {
    SERQ_CUDA(cudaFuncSetAttribute(producer_quant_kernel<KIND, FMT, MAXC>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, 4 * 32768));
    return SERQ_OK;
}

serq_status producer_setup(DeviceInfo* info) {
    if (info->smem_set_prod) return SERQ_OK;
    serq_status st = producer_setup_one<0, 0, 8>();
    if (!st) st = producer_setup_one<0, 0, 16>();
    if (!st) st = producer_setup_one<0, 1, 1>();
    if (!st) st = producer_setup_one<0, 2, 8>();
    if (!st) st = producer_setup_one<0, 2, 16>();
    if (!st) st = producer_setup_one<1, 0, 8>();
    if (!st) st = producer_setup_one<1, 0, 16>();
    if (!st) st = producer_setup_one<1, 1, 1>();
    if (!st) st = producer_setup_one<1, 2, 8>();
    if (!st) st = producer_setup_one<1, 2, 16>();
    if (!st) st = producer_setup_one<2, 0, 8>();
    if (!st) st = producer_setup_one<2, 0, 16>();
    if (!st) st = producer_setup_one<2, 1, 1>();
    if (!st) st = producer_setup_one<2, 2, 8>();
    if (!st) st = producer_setup_one<2, 2, 16>();
    if (!st) info->smem_set_prod = true;
    return st;
}

// Shared checks and launch of the fused producer + quantization kernels.
serq_status producer_launch(int kind, const serq_weight* w, const void* in, const void* gamma, float eps, int M,
                            void* xq, void* xs, void* xsq, void* xss, void* xhat, serq_stream stream) {
    if (w == nullptr || in == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    if (M < 1) return fail(SERQ_EINVAL, "M must be >= 1");
    if (kind == 0 && (gamma == nullptr || !aligned16(gamma))) return fail(SERQ_EINVAL, "gamma must be a 16-byte aligned pointer");
    if (kind == 0 && !(eps >= 0.0f && std::isfinite(eps))) return fail(SERQ_EINVAL, "eps must be finite and >= 0");
    if (xq == nullptr || xs == nullptr) return fail(SERQ_EINVAL, "NULL output");
    if (w->rp > 0 && (xsq == nullptr || xss == nullptr)) return fail(SERQ_EINVAL, "r > 0 needs xsq and xss");
    if (!aligned16(in) || !aligned16(xq) || !aligned16(xs) || !aligned16(xhat) ||
        (w->rp > 0 && (!aligned16(xsq) || !aligned16(xss))))
        return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    if (dev != w->device) return fail(SERQ_EINVAL, "weight lives on device %d, current device is %d", w->device, dev);
    if (serq_status st = producer_setup(info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    ProducerParams p;
    p.K = w->K;
    p.r = w->r;
    p.rp = w->rp;
    p.perm = w->perm;
    p.inv_s = w->inv_s;
    p.s_perm = w->s_perm;
    p.gamma = static_cast<const __nv_bfloat16*>(gamma);
    p.eps = eps;
    p.xq = xq;
    p.xs = xs;
    p.xsq = xsq;
    p.xss = xss;
    p.xhat = static_cast<__nv_bfloat16*>(xhat);
    const uint4* src = static_cast<const uint4*>(in);
    const size_t smem = static_cast<size_t>(w->K) * (kind == 1 ? 4 : 2);
    const bool wide = w->K > 16384;
    const int f = w->fmt;
#define SERQ_PRODUCER(KIND)                                                                        \
    do {                                                                                           \
        if (f == SERQ_FMT_MXFP4)                                                                   \
            producer_quant_kernel<KIND, 1, 1><<<M, kQuantThreads, smem, cs>>>(src, p);            \
        else if (f == SERQ_FMT_INT4)                                                               \
            (wide ? producer_quant_kernel<KIND, 0, 16> : producer_quant_kernel<KIND, 0, 8>)        \
                <<<M, kQuantThreads, smem, cs>>>(src, p);                                          \
        else                                                                                       \
            (wide ? producer_quant_kernel<KIND, 2, 16> : producer_quant_kernel<KIND, 2, 8>)        \
                <<<M, kQuantThreads, smem, cs>>>(src, p);                                          \
    } while (0)
    if (kind == 0)
        SERQ_PRODUCER(0);
    else if (kind == 1)
        SERQ_PRODUCER(1);
    else
        SERQ_PRODUCER(2);
#undef SERQ_PRODUCER
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

// CTA-pair MXFP4 kernel (M > 128): tile set-up and launch; `p` carries the
// epilogue's outputs (Y, or for EPI = 1 the SwiGLU outputs).
template <int EPI>
serq_status launch_pair(const serq_weight* w, DeviceInfo* info, int M, const CUtensorMap& tm_a, const CUtensorMap& tm_ar,
                        const void* xs, const void* xss, MxPairParams p, cudaStream_t cs) {
    const int K = w->K, N = w->N, rp = w->rp;
    if (!info->smem_set_mxp) {
        SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_pair_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       mxp::SMEM_BYTES));
        SERQ_CUDA(cudaFuncSetAttribute(serq_linear_mxfp4_pair_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
        if (cudaOccupancyMaxActiveClusters(&n, serq_linear_mxfp4_pair_kernel<0>, &qc) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = info->sms / 2;
        }
        info->pair_clusters = n;
        info->smem_set_mxp = true;
    }
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
    const size_t row_blocks_a = static_cast<size_t>((M + 127) / 128);
    MxPairScaleMaps sf;
    if (serq_status st = make_sfa_wide_map(&sf.sfa, xs, row_blocks_a * p.atoms_k_main * 512)) return st;
    sf.sfb = w->tm_wsf;
    if (rp > 0) {
        if (serq_status st = make_sfa_wide_map(&sf.sfa_r, xss, row_blocks_a * p.atoms_k_res * 512)) return st;
    } else {
        sf.sfa_r = sf.sfa;
    }
    sf.sfb_r = w->tm_rsf;
    const int pairs = info->pair_clusters;
    const int grid2 = 2 * (p.num_tiles < pairs ? p.num_tiles : pairs);
    serq_linear_mxfp4_pair_kernel<EPI><<<grid2, mxp::THREADS, mxp::SMEM_BYTES, cs>>>(tm_a, w->tm_w128, tm_ar,
                                                                                    w->tm_r128, sf, p);
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

}  // namespace

extern "C" {

serq_status serq_rmsnorm_quant_act(const serq_weight* w, const void* H, const void* gamma, float eps, int M, void* xq,
                                   void* xs, void* xsq, void* xss, void* xhat, serq_stream stream) {
    return producer_launch(0, w, H, gamma, eps, M, xq, xs, xsq, xss, xhat, stream);
}

serq_status serq_swiglu_quant_act(const serq_weight* w, const void* Ygu, int M, void* xq, void* xs, void* xsq,
                                  void* xss, void* xhat, serq_stream stream) {
    return producer_launch(1, w, Ygu, nullptr, 0.0f, M, xq, xs, xsq, xss, xhat, stream);
}

serq_status serq_fold_quant_act(const serq_weight* w, const void* X, int M, void* xq, void* xs, void* xsq, void* xss,
                                void* xhat, serq_stream stream) {
    return producer_launch(2, w, X, nullptr, 0.0f, M, xq, xs, xsq, xss, xhat, stream);
}

serq_status serq_rope(void* x, int M, int ld, int n_heads, int head_dim, float base, int pos0, serq_stream stream) {
    if (x == nullptr || !aligned16(x)) return fail(SERQ_EINVAL, "x must be a 16-byte aligned pointer");
    if (M < 1 || n_heads < 1 || head_dim < 2 || head_dim % 2 != 0 || ld < n_heads * head_dim || !(base > 1.0f) ||
        pos0 < 0)
        return fail(SERQ_EINVAL, "bad RoPE arguments M=%d ld=%d heads=%d dim=%d", M, ld, n_heads, head_dim);
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const size_t n = static_cast<size_t>(M) * n_heads * (head_dim / 2);
    rope_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, cs>>>(static_cast<__nv_bfloat16*>(x), M, ld, n_heads,
                                                                        head_dim, log2f(base), pos0);
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

serq_status serq_attention_prefill(const void* q, int ldq, const void* k, const void* v, int ldkv, int M, int n_q,
                                   int n_kv, int head_dim, void* o, int ldo, serq_stream stream) {
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return fail(SERQ_EINVAL, "NULL pointer");
    if (head_dim != atc::D) return fail(SERQ_EUNSUPPORTED, "head_dim %d (only %d)", head_dim, atc::D);
    if (M < 1 || n_q < 1 || n_kv < 1 || n_q % n_kv != 0) return fail(SERQ_EINVAL, "bad M / head counts");
    if (ldq < n_q * head_dim || ldkv < n_kv * head_dim || ldo < n_q * head_dim || ldq % 8 || ldkv % 8 || ldo % 8)
        return fail(SERQ_EINVAL, "leading dimensions must cover the heads and be multiples of 8");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    SERQ_CUDA(cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   atc::SMEM_BYTES));
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    // V^T of each key-value group (dims x keys), the second product's K-major B operand;
    // stream-ordered scratch
    const int M_pad = (M + 63) / 64 * 64;
    const size_t vt_bytes = static_cast<size_t>(n_kv) * head_dim * M_pad * sizeof(__nv_bfloat16);
    void* vt = nullptr;
    cudaMemPool_t pool;
    if (serq_status pst = scratch_pool(dev, info, &pool)) return pst;
    SERQ_CUDA(cudaMallocFromPoolAsync(&vt, vt_bytes, pool, cs));
    transpose_v_kernel<<<dim3(M_pad / 32, n_kv * head_dim / 32), dim3(32, 8), 0, cs>>>(
        static_cast<const __nv_bfloat16*>(v), ldkv, M, M_pad, static_cast<__nv_bfloat16*>(vt));
    serq_status st = SERQ_OK;
    const cudaError_t le = cudaGetLastError();
    if (le != cudaSuccess) st = cuda_fail(le, "transpose_v_kernel");
    CUtensorMap tm_q, tm_k, tm_vt;
    if (!st) st = make_map(&tm_q, q, static_cast<uint64_t>(ldq) * 2, M, 128, atc::BM, true);
    if (!st) st = make_map(&tm_k, k, static_cast<uint64_t>(ldkv) * 2, M, 128, atc::BN, true);
    if (!st) st = make_map(&tm_vt, vt, static_cast<uint64_t>(M_pad) * 2, static_cast<uint64_t>(n_kv) * head_dim, 128, atc::D, true);
    if (!st) {
        AttTcParams p;
        p.M = M;
        p.n_q = n_q;
        p.n_kv = n_kv;
        p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(head_dim));
        p.o = static_cast<__nv_bfloat16*>(o);
        p.ldo = ldo;
        attention_tc_kernel<<<dim3((M + atc::BM - 1) / atc::BM, n_q), atc::THREADS, atc::SMEM_BYTES, cs>>>(tm_q, tm_k,
                                                                                                       tm_vt, p);
        const cudaError_t ke = cudaGetLastError();
        if (ke != cudaSuccess) st = cuda_fail(ke, "attention_tc_kernel");
    }
    const cudaError_t fe = cudaFreeAsync(vt, cs);
    if (!st && fe != cudaSuccess) st = cuda_fail(fe, "cudaFreeAsync");
    return st;
}

serq_status serq_add(const void* a, const void* b, void* out, size_t n, serq_stream stream) {
    if (a == nullptr || b == nullptr || out == nullptr || n % 8 != 0)
        return fail(SERQ_EINVAL, "NULL pointer or n not a multiple of 8");
    if (!aligned16(a) || !aligned16(b) || !aligned16(out)) return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const size_t n8 = n / 8;
    if (n8 > 0)
        add_bf16_kernel<<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, cs>>>(
            static_cast<const uint4*>(a), static_cast<const uint4*>(b), static_cast<uint4*>(out), n8);
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
    if (acc_dbg != nullptr && !int_weights(w->fmt)) return fail(SERQ_EINVAL, "acc_dbg needs INT4 weights");
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

    CUtensorMap tm_a, tm_ar;
    if (w->fmt == SERQ_FMT_W4A8) {
        // int8 activations: 128-byte rows of a K-tile, swizzled straight into the MMA layout
        if (serq_status st = make_map(&tm_a, xq, K, M, 128, 128, true)) return st;
        if (rp > 0) {
            if (serq_status st = make_map(&tm_ar, xsq, rp, M, 128, 128, true)) return st;
        } else {
            tm_ar = tm_a;
        }
    } else {
        const uint32_t bi = box_inner_bytes(w->fmt);
        const bool swz = w->fmt == SERQ_FMT_MXFP4;
        if (serq_status st = make_map(&tm_a, xq, K / 2, M, bi, 128, swz)) return st;
        if (rp > 0) {
            if (serq_status st = make_map(&tm_ar, xsq, rp / 2, M, bi, 128, swz)) return st;
        } else {
            tm_ar = tm_a;
        }
    }
    const int num_m = (M + 127) / 128;
    const int num_n = (N + 255) / 256;
    const int tiles = num_m * num_n;
    const int grid = tiles < info->sms ? tiles : info->sms;

    if (w->fmt == SERQ_FMT_MXFP4 && M > 128) {
        // CTA-pair kernel: 256 x 256 tiles, B halves split across the pair
        MxPairParams p{};
        p.Y = static_cast<__nv_bfloat16*>(Y);
        if (serq_status st = launch_pair<0>(w, info, M, tm_a, tm_ar, xs, xss, p, cs)) return st;
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
            SERQ_CUDA(cudaFuncSetAttribute(serq_linear_int4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           i4::Plan<false>::SMEM_BYTES));
            SERQ_CUDA(cudaFuncSetAttribute(serq_linear_int4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           i4::Plan<true>::SMEM_BYTES));
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
        if (w->fmt == SERQ_FMT_W4A8)
            serq_linear_int4_kernel<true><<<grid, i4::THREADS, i4::Plan<true>::SMEM_BYTES, cs>>>(tm_a, w->tm_w, tm_ar,
                                                                                               w->tm_r, p);
        else
            serq_linear_int4_kernel<false><<<grid, i4::THREADS, i4::Plan<false>::SMEM_BYTES, cs>>>(tm_a, w->tm_w, tm_ar,
                                                                                                 w->tm_r, p);
    }
    SERQ_CUDA(cudaGetLastError());
    return SERQ_OK;
}

serq_status serq_prepare_swiglu(const serq_prepare_desc* gate_up, const serq_weight* down, serq_weight** out,
                                serq_stream stream) {
    if (gate_up == nullptr || down == nullptr || out == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    *out = nullptr;
    if (gate_up->fmt != SERQ_FMT_MXFP4 || down->fmt != SERQ_FMT_MXFP4)
        return fail(SERQ_EUNSUPPORTED, "the fused SwiGLU epilogue is MXFP4 only");
    const int F = down->K;
    if (gate_up->N != 2 * F) return fail(SERQ_EINVAL, "gate/up N=%d must be 2 x down's K=%d", gate_up->N, F);
    if (gate_up->R != nullptr) return fail(SERQ_EINVAL, "a given residual is not supported here");
    if (serq_status st = check_weight_shape(gate_up->K, gate_up->N, gate_up->r, gate_up->fmt)) return st;
    if (gate_up->W == nullptr || !aligned16(gate_up->W)) return fail(SERQ_EINVAL, "W must be a 16-byte aligned pointer");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    if (dev != down->device) return fail(SERQ_EINVAL, "down lives on device %d, current device is %d", down->device, dev);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const size_t elems = static_cast<size_t>(gate_up->K) * gate_up->N;
    void* wp = nullptr;
    float* inv = nullptr;
    int pending = g_fail_allocs.load();
    while (pending > 0 && !g_fail_allocs.compare_exchange_weak(pending, pending - 1)) {
    }
    if (pending > 0) return fail(SERQ_ENOMEM, "device allocation failed (injected by the test hook)");
    if (cudaMalloc(&wp, elems * 2) != cudaSuccess) {
        cudaGetLastError();
        return fail(SERQ_ENOMEM, "cudaMalloc(%zu) for the arranged gate/up weight failed", elems * 2);
    }
    if (cudaMalloc(reinterpret_cast<void**>(&inv), sizeof(float) * F) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(wp);
        return fail(SERQ_ENOMEM, "cudaMalloc of down's 1/s failed");
    }
    auto cleanup = [&](serq_status st) {
        cudaStreamSynchronize(cs);
        cudaFree(wp);
        if (inv != nullptr) cudaFree(inv);
        return st;
    };
    swiglu_arrange_kernel<<<static_cast<unsigned>((elems + 255) / 256), 256, 0, cs>>>(
        static_cast<const __nv_bfloat16*>(gate_up->W), gate_up->K, F, down->perm, static_cast<__nv_bfloat16*>(wp));
    if (cudaError_t e = cudaGetLastError()) return cleanup(cuda_fail(e, "swiglu_arrange_kernel"));
    if (cudaError_t e = cudaMemcpyAsync(inv, down->inv_s, sizeof(float) * F, cudaMemcpyDeviceToDevice, cs))
        return cleanup(cuda_fail(e, "cudaMemcpyAsync(down 1/s)"));
    serq_prepare_desc d = *gate_up;
    d.W = wp;
    serq_weight* w = nullptr;
    if (serq_status st = serq_prepare(&d, &w, stream)) return cleanup(st);  // synchronizes
    cudaFree(wp);
    w->swiglu_inv_s = inv;
    w->swiglu_F = F;
    w->swiglu_r = down->r;
    w->swiglu_rp = down->rp;
    *out = w;
    return SERQ_OK;
}

serq_status serq_linear_swiglu_quant(const serq_weight* w, int M, const void* xq, const void* xs, const void* xsq,
                                     const void* xss, void* hq, void* hs, void* hsq, void* hss, void* xhat,
                                     serq_stream stream) {
    if (w == nullptr) return fail(SERQ_EINVAL, "weight is NULL");
    if (w->swiglu_F == 0) return fail(SERQ_EINVAL, "the weight was not prepared by serq_prepare_swiglu");
    if (M <= 128) return fail(SERQ_EUNSUPPORTED, "the fused SwiGLU epilogue needs M > 128 (M=%d)", M);
    if (xq == nullptr || xs == nullptr || hq == nullptr || hs == nullptr) return fail(SERQ_EINVAL, "NULL pointer");
    if (w->rp > 0 && (xsq == nullptr || xss == nullptr)) return fail(SERQ_EINVAL, "r > 0 needs xsq and xss");
    if (w->swiglu_rp > 0 && (hsq == nullptr || hss == nullptr)) return fail(SERQ_EINVAL, "down's r > 0 needs hsq and hss");
    if (!aligned16(xq) || !aligned16(xs) || !aligned16(hq) || !aligned16(hs) || !aligned16(xhat) ||
        (w->rp > 0 && (!aligned16(xsq) || !aligned16(xss))) || (w->swiglu_rp > 0 && (!aligned16(hsq) || !aligned16(hss))))
        return fail(SERQ_EINVAL, "pointers must be 16-byte aligned");
    int dev;
    DeviceInfo* info;
    if (serq_status st = device_check(&dev, &info)) return st;
    if (dev != w->device) return fail(SERQ_EINVAL, "weight lives on device %d, current device is %d", w->device, dev);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int K = w->K, rp = w->rp;
    CUtensorMap tm_a, tm_ar;
    if (serq_status st = make_map(&tm_a, xq, K / 2, M, 128, 128, true)) return st;
    if (rp > 0) {
        if (serq_status st = make_map(&tm_ar, xsq, rp / 2, M, 128, 128, true)) return st;
    } else {
        tm_ar = tm_a;
    }
    MxPairParams p{};
    p.F = w->swiglu_F;
    p.r_d = w->swiglu_r;
    p.rp_d = w->swiglu_rp;
    p.inv_s_d = w->swiglu_inv_s;
    p.hq = static_cast<uint32_t*>(hq);
    p.hs = static_cast<uint8_t*>(hs);
    p.hsq = static_cast<uint32_t*>(hsq);
    p.hss = static_cast<uint8_t*>(hss);
    p.xhat = static_cast<__nv_bfloat16*>(xhat);
    return launch_pair<1>(w, info, M, tm_a, tm_ar, xs, xss, p, cs);
}

serq_status serq_linear_l2qer(const serq_weight* main, const serq_weight* l1, int M, const void* xq, const void* xs,
                              void* T, void* tq, void* ts, void* tsq, void* tss, void* Y, serq_stream stream) {
    if (main == nullptr || l1 == nullptr || T == nullptr) return fail(SERQ_EINVAL, "NULL argument");
    if (l1->r != 0 || l1->K != main->K || l1->N != main->r || l1->fmt != main->fmt)
        return fail(SERQ_EINVAL, "l1 must be K x k with r = 0 and main's format, k = main's r (%d)", main->r);
    // T = X_q L1_q (bf16), then Q(T) on the fly, then X_q W_q + Q(T) L2_q in one launch
    if (serq_status st = serq_linear(l1, M, xq, xs, nullptr, nullptr, T, nullptr, stream)) return st;
    const int k = main->r;
    if (serq_status st = serq_quant_act(T, M, k, k, main->fmt, tq, ts, tsq, tss, stream)) return st;
    return serq_linear(main, M, xq, xs, tsq, tss, Y, nullptr, stream);
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
