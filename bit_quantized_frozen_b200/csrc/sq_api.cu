// sq_api.cu -- the C ABI of libsq (include/sq.h): host-side validation,
// workspace carving and the launch sequence of each operation.  Nothing here
// allocates, synchronises or copies to the host (except the explicit status
// read-back); every error is returned as an sq_status before any launch.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <cstdio>
#include <cstring>

#include "sq.h"
#include "sq_device.cuh"
#include "sq_kernels.h"
#include "sq_ptx.cuh"

static __device__ __align__(256) uint8_t g_noalloc_scratch[size_t(96) << 20];

namespace sq {
typedef CUresult (*PFN_ctxGetCurrent)(CUcontext *);
typedef CUresult (*PFN_ctxGetId)(CUcontext, unsigned long long *);

unsigned long long current_context_id()
{
    static PFN_ctxGetCurrent get_current = nullptr;
    static PFN_ctxGetId get_id = nullptr;
    if (!get_current || !get_id) {
        void *p = nullptr, *q = nullptr;
        cudaDriverEntryPointQueryResult r1, r2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) != cudaSuccess ||
            r1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) != cudaSuccess ||
            r2 != cudaDriverEntryPointSuccess)
            return 0;
        get_current = reinterpret_cast<PFN_ctxGetCurrent>(p);
        get_id = reinterpret_cast<PFN_ctxGetId>(q);
    }
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

}  // namespace sq


// One thread checks the index one past `bound` with the device-side index check
// of the debug builds: the check fails, the access it guards (never made) is
// skipped, and the status word gets the index bit.
static __global__ void selftest_index_kernel(uint32_t *status, uint32_t bound)
{
    if (threadIdx.x == 0) {
        const uint32_t idx = bound;
        if (sq::dcheck(idx < bound, status))
            status[1] = idx;                          // unreachable: the check fails
    }
}

// One thread waits on an mbarrier that nothing ever arrives on, with the
// bounded wait every kernel of the library uses; it must give up after
// limit_ns, set the status word and return.
static __global__ void selftest_wait_kernel(uint32_t *status, unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        sq::mbar_init(sq::smem_u32(&bar), 1);
        abort_flag = 0u;
        sq::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        (void)sq::mbar_wait(sq::smem_u32(&bar), 0u, &abort_flag, status, limit_ns);
}

namespace {

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];          // 0 = not yet queried
int g_cc_ok[kMaxDevices];        // 0 unknown, 1 sm_100, -1 other

thread_local char g_detail[256] = "";
// sq_set_stage_events: [stage][0 = before the launch, 1 = after]
thread_local cudaEvent_t g_stage_ev[SQ_STAGE_COUNT][2] = {};

// record stage event `which` (0 before, 1 after) on stream s, when the caller set one
cudaError_t stage_event(int stage, int which, cudaStream_t s)
{
    cudaEvent_t e = g_stage_ev[stage][which];
    return e ? cudaEventRecord(e, s) : cudaSuccess;
}

void set_detail(const char *what, cudaError_t e)
{
    snprintf(g_detail, sizeof(g_detail), "%s: %s", what, cudaGetErrorString(e));
}

// current device must be compute capability 10.0 (the sm_100a code this library carries)
sq_status check_device(int *sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_detail("cudaGetDevice", e);
        return SQ_ERR_DEVICE;
    }
    if (dev < 0 || dev >= kMaxDevices)
        return SQ_ERR_DEVICE;
    if (g_cc_ok[dev] == 0) {
        int major = 0, minor = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SQ_ERR_DEVICE;
        g_sms[dev] = n;
        g_cc_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    if (g_cc_ok[dev] != 1) {
        snprintf(g_detail, sizeof(g_detail), "device %d is not compute capability 10.0", dev);
        return SQ_ERR_DEVICE;
    }
    *sms = g_sms[dev];
    return SQ_OK;
}

bool aligned(const void *p, uintptr_t a)
{
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

size_t round_up(size_t v, size_t a)
{
    return (v + a - 1) / a * a;
}

constexpr int64_t kMaxM = int64_t(1) << 24;
constexpr int64_t kMaxN = int64_t(1) << 20;
constexpr int64_t kMaxK = int64_t(1) << 17;
constexpr int64_t kMaxKInt8 = 16384;          // the int8 builder keeps one rotated row in shared memory

bool shape_ok_nk(int64_t N, int64_t K)
{
    return N >= 128 && N % 128 == 0 && N <= kMaxN && K >= 256 && K % 256 == 0 && K <= kMaxK;
}

bool shape_ok_mk(int64_t M, int64_t K)
{
    return M >= 1 && M <= kMaxM && K >= 256 && K % 256 == 0 && K <= kMaxK;
}

// workspace layout ----------------------------------------------------------
// [0, 256): header -- u32 status, u32 amax, f32 g_x scratch
constexpr size_t kHeader = 256;
constexpr size_t kAlign = 1024;

struct FwdLayout {
    size_t a = 0, a_sf = 0, t32 = 0, tsplit = 0, udup = 0, d32 = 0, u32 = 0, ring = 0, ring_ctr = 0, total = 0;
};

// slots of the int4 / int8 GEMM's W ring: the W tiles in flight at once (the GEMM's CTA
// pairs -- 74 on a B200 -- spread over m_tiles clusters per W tile) plus two for the
// writers to run ahead, never more than there are W tiles.  Fewer slots would still be
// correct (every wait points at an earlier W tile) but would make tiles wait in turn.
constexpr int64_t kGemmPairs = 74;
int64_t ring_slots(int64_t M, int64_t N)
{
    const int64_t m_tiles = (M + 255) / 256, n_tiles = (N + 255) / 256;
    const int64_t want = (kGemmPairs + m_tiles - 1) / m_tiles + 2;
    return want < n_tiles ? want : n_tiles;
}

FwdLayout fwd_layout(int fmt, int64_t M, int64_t N, int64_t K)
{
    FwdLayout L;
    size_t off = kHeader;
    auto take = [&](size_t bytes) {
        off = round_up(off, kAlign);
        size_t at = off;
        off += bytes;
        return at;
    };
    if (fmt == SQ_FMT_NVFP4) {
        L.a = take((size_t)M * (size_t)K / 2);
        L.a_sf = take(sq_sf_bytes(M, K));
    } else {
        L.a = take((size_t)M * (size_t)K * 2);    // bf16(H x)
        // the GEMM's ring of dequantised 256-row W tiles, and its counters
        L.ring = take((size_t)ring_slots(M, N) * 256 * (size_t)K * 2);
        L.ring_ctr = take((size_t)2 * ring_slots(M, N) * 4);
    }
    L.t32 = take((size_t)sq::act_t_parts(M, K) * (size_t)M * 32 * 4);   // partial tiles of t
    L.tsplit = take((size_t)M * 64 * 2);
    L.udup = take((size_t)N * 64 * 2);
    if (fmt == SQ_FMT_INT8_ROW) {                 // rank-16 factors widened to rank 32
        L.d32 = take((size_t)K * 32 * 2);
        L.u32 = take((size_t)N * 32 * 2);
    }
    L.total = round_up(off, kAlign);
    return L;
}

uint8_t *ws_at(void *ws, size_t off)
{
    return reinterpret_cast<uint8_t *>(ws) + off;
}

#define SQ_CUDA(call, what)                     \
    do {                                        \
        cudaError_t e_ = (call);                \
        if (e_ != cudaSuccess) {                \
            set_detail(what, e_);               \
            return SQ_ERR_CUDA;                 \
        }                                       \
    } while (0)

// Static scratch of sq_linear_fwd_noalloc --------------------------------------
// A fixed 96 MiB forward workspace that lives in the module's own device
// memory (one copy per device, created when the module's device code is
// loaded into a context, released with the context), so that the call needs
// no allocation.  Its device address is looked up with the device current,
// once per device and context: the address is kept together with the ID of
// the context it was looked up in, and looked up again when the current
// context has another ID (after cudaDeviceReset, or once the primary context
// was released and created again, the module is loaded anew and the array may
// sit elsewhere).
constexpr size_t kNoAllocScratchBytes = size_t(96) << 20;
struct ScratchSlot {
    void *ptr = nullptr;
    unsigned long long ctx = 0;
};
ScratchSlot g_noalloc_scratch_slot[kMaxDevices];
std::mutex g_noalloc_mutex;

sq_status check_weight(const sq_weight *w)
{
    if (!w || !w->codes || !w->scales)
        return SQ_ERR_NULL;
    if (w->fmt != SQ_FMT_INT4_G32 && w->fmt != SQ_FMT_NVFP4 && w->fmt != SQ_FMT_INT4_G64 &&
        w->fmt != SQ_FMT_INT8_ROW)
        return SQ_ERR_ARG;
    if (w->fmt == SQ_FMT_NVFP4 && !w->g_w)
        return SQ_ERR_NULL;
    if (!shape_ok_nk(w->N, w->K) || (w->fmt == SQ_FMT_INT8_ROW && w->K > kMaxKInt8))
        return SQ_ERR_SHAPE;
    if (!aligned(w->codes, 16) || !aligned(w->scales, 16) || !aligned(w->g_w, 4) ||
        !aligned(w->lora_up, 16) || !aligned(w->lora_down, 16))
        return SQ_ERR_ALIGN;
    return SQ_OK;
}

}  // namespace

extern "C" {

const char *sq_status_str(int status)
{
    switch (status) {
    case SQ_OK: return "ok";
    case SQ_ERR_NULL: return "null pointer";
    case SQ_ERR_SHAPE: return "unsupported shape";
    case SQ_ERR_ALIGN: return "misaligned pointer";
    case SQ_ERR_WORKSPACE: return "workspace too small";
    case SQ_ERR_DEVICE: return "device is not sm_100";
    case SQ_ERR_CUDA: return "CUDA error";
    case SQ_ERR_ARG: return "bad argument";
    case SQ_ERR_TIMEOUT: return "kernel wait timed out";
    case SQ_ERR_NONFINITE: return "non-finite input";
    case SQ_ERR_INDEX: return "device index check failed";
    default: return "unknown status";
    }
}

int sq_abi_version(void)
{
    return 1;
}

int sq_debug_checks(void)
{
#ifdef SQ_DEBUG_CHECKS
    return 1;
#else
    return 0;
#endif
}

const char *sq_last_error_detail(void)
{
    return g_detail;
}

size_t sq_sf_bytes(int64_t rows, int64_t K)
{
    if (rows < 0 || K < 0)
        return 0;
    return (size_t)((rows + 127) / 128 * 128) * (size_t)(K / 16);
}

size_t sq_workspace_bytes(int op, int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K < 0)
        return 0;
    switch (op) {
    case SQ_OP_BUILD_INT4:
    case SQ_OP_RECONSTRUCT:
        return kHeader;
    case SQ_OP_BUILD_NVFP4:
        return kHeader;
    case SQ_OP_ACT_QUANT_NVFP4: {
        // the partial tiles of t = x lora_down when K is split over several CTAs
        const int parts = sq::act_t_parts(M, K);
        return parts > 1 ? kAlign + round_up((size_t)parts * (size_t)M * 32 * 4, kAlign) : kHeader;
    }
    case SQ_OP_LINEAR_FWD_NVFP4:
        return fwd_layout(SQ_FMT_NVFP4, M, N, K).total;
    case SQ_OP_LINEAR_FWD_INT4:
        return fwd_layout(SQ_FMT_INT4_G32, M, N, K).total;
    case SQ_OP_LINEAR_FWD_INT8:
        return fwd_layout(SQ_FMT_INT8_ROW, M, N, K).total;
    case SQ_OP_BUILD_INT8:
        return kHeader;
    case SQ_OP_LINEAR_BWD_DX:
        return kAlign + round_up((size_t)N * (size_t)K * 2, kAlign);
    case SQ_OP_SVD_INIT:
        return sq::svd_workspace_bytes(N, K);
    default:
        return 0;
    }
}

sq_status sq_build_int4(const float *R, int64_t N, int64_t K, int32_t group, uint8_t *codes, uint16_t *scales,
                        uint8_t *frac_idx, void *stream)
{
    if (!R || !codes || !scales)
        return SQ_ERR_NULL;
    if ((group != 32 && group != 64) || !shape_ok_nk(N, K))
        return SQ_ERR_SHAPE;
    if (!aligned(R, 16) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(frac_idx, 16))
        return SQ_ERR_ALIGN;
    int sms = 0;
    sq_status st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    SQ_CUDA(sq::launch_int4_build(R, N, K, group, codes, scales, frac_idx, sms, s), "int4 build");
    return SQ_OK;
}

sq_status sq_build_int8(const float *R, int64_t N, int64_t K, int8_t *codes, float *scales, uint8_t *frac_idx,
                        void *stream)
{
    if (!R || !codes || !scales)
        return SQ_ERR_NULL;
    if (!shape_ok_nk(N, K) || K > kMaxKInt8)
        return SQ_ERR_SHAPE;
    if (!aligned(R, 16) || !aligned(codes, 16) || !aligned(scales, 4))
        return SQ_ERR_ALIGN;
    int sms = 0;
    sq_status st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    SQ_CUDA(sq::launch_int8_build(R, N, K, codes, scales, frac_idx, sms, s), "int8 build");
    return SQ_OK;
}

sq_status sq_svd_init(const float *W, int64_t N, int64_t K, const float *omega, int32_t iters, int32_t rank,
                      uint16_t *lora_up, uint16_t *lora_down, float *R, void *ws, size_t ws_bytes, void *stream)
{
    if (!W || !omega || !lora_up || !lora_down || !R || !ws)
        return SQ_ERR_NULL;
    if (!shape_ok_nk(N, K))
        return SQ_ERR_SHAPE;
    if (iters < 1 || iters > 100 || (rank != 16 && rank != 32))
        return SQ_ERR_ARG;
    if (!aligned(W, 16) || !aligned(omega, 16) || !aligned(lora_up, 16) || !aligned(lora_down, 16) ||
        !aligned(R, 16) || !aligned(ws, 256))
        return SQ_ERR_ALIGN;
    if (ws_bytes < sq_workspace_bytes(SQ_OP_SVD_INIT, 0, N, K))
        return SQ_ERR_WORKSPACE;
    int sms = 0;
    sq_status st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const char *stage = "svd init";
    const cudaError_t e =
        sq::launch_svd_init(W, N, K, omega, iters, rank, lora_up, lora_down, R, ws, sms, s, &stage);
    if (e != cudaSuccess) {
        set_detail(stage, e);
        return SQ_ERR_CUDA;
    }
    return SQ_OK;
}

sq_status sq_build_nvfp4(const float *R, int64_t N, int64_t K, uint8_t *codes, uint8_t *sf_tiled, float *g_w,
                         void *ws, size_t ws_bytes, void *stream)
{
    if (!R || !codes || !sf_tiled || !g_w || !ws)
        return SQ_ERR_NULL;
    if (!shape_ok_nk(N, K))
        return SQ_ERR_SHAPE;
    if (!aligned(R, 16) || !aligned(codes, 16) || !aligned(sf_tiled, 16) || !aligned(g_w, 4) || !aligned(ws, 256))
        return SQ_ERR_ALIGN;
    if (ws_bytes < sq_workspace_bytes(SQ_OP_BUILD_NVFP4, 0, N, K))
        return SQ_ERR_WORKSPACE;
    int sms = 0;
    sq_status st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *amax = reinterpret_cast<uint32_t *>(ws_at(ws, 4));
    SQ_CUDA(cudaMemsetAsync(amax, 0, 4, s), "memset");
    SQ_CUDA(sq::launch_absmax_rot_f32(R, N, K, amax, sms, s), "absmax");
    SQ_CUDA(sq::launch_nvfp4_quant_f32(R, N, K, amax, nullptr, g_w, codes, sf_tiled, sms, s), "nvfp4 quant");
    return SQ_OK;
}

sq_status sq_act_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K, uint8_t *codes, uint8_t *sf_tiled,
                             float *g_x, const uint16_t *lora_down, float *t, uint32_t flags, void *ws,
                             size_t ws_bytes, void *stream)
{
    if (!x || !codes || !sf_tiled || !g_x || !ws)
        return SQ_ERR_NULL;
    if (flags & ~(SQ_ACT_STATIC_SCALE | SQ_CHECK_FINITE))
        return SQ_ERR_ARG;
    if (!shape_ok_mk(M, K))
        return SQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(sf_tiled, 16) || !aligned(g_x, 4) ||
        !aligned(lora_down, 16) || !aligned(t, 16) || !aligned(ws, 256))
        return SQ_ERR_ALIGN;
    if (ws_bytes < sq_workspace_bytes(SQ_OP_ACT_QUANT_NVFP4, M, 0, K))
        return SQ_ERR_WORKSPACE;
    int sms = 0;
    sq_status st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool stat = (flags & SQ_ACT_STATIC_SCALE) != 0;
    const bool with_t = lora_down && t;
    const int parts = sq::act_t_parts(M, K);
    float *t_part = !with_t ? nullptr : parts > 1 ? reinterpret_cast<float *>(ws_at(ws, kAlign)) : t;
    uint32_t *amax = reinterpret_cast<uint32_t *>(ws_at(ws, 4));
    SQ_CUDA(cudaMemsetAsync(ws, 0, 8, s), "memset");          // status word + absmax
    if (flags & SQ_CHECK_FINITE)
        SQ_CUDA(sq::launch_check_finite_bf16(x, M * K, reinterpret_cast<uint32_t *>(ws), sms, s), "finite check");
    if (!stat || with_t) {
        SQ_CUDA(stage_event(SQ_STAGE_ACT_PASS1, 0, s), "event record");
        SQ_CUDA(sq::launch_act_pass1(x, M, K, lora_down, stat ? nullptr : amax, t_part, nullptr,
                                     reinterpret_cast<uint32_t *>(ws), sms, s),
                "activation pass 1");
        SQ_CUDA(stage_event(SQ_STAGE_ACT_PASS1, 1, s), "event record");
    }
    sq::LowrankOut lr;                                          // t = the sum of the partial tiles
    if (with_t && parts > 1) {
        lr.t_part = t_part;
        lr.parts = parts;
        lr.t_out = t;
    }
    SQ_CUDA(stage_event(SQ_STAGE_ACT_QUANT, 0, s), "event record");
    SQ_CUDA(sq::launch_nvfp4_quant_bf16(x, M, K, amax, stat ? g_x : nullptr, stat ? nullptr : g_x, codes, sf_tiled,
                                        lr, reinterpret_cast<uint32_t *>(ws), sms, s),
            "nvfp4 quant");
    SQ_CUDA(stage_event(SQ_STAGE_ACT_QUANT, 1, s), "event record");
    return SQ_OK;
}

sq_status sq_linear_fwd(const sq_weight *w, const uint16_t *x, int64_t M, void *y, float *g_x, uint32_t flags,
                        void *ws, size_t ws_bytes, void *stream)
{
    sq_status st = check_weight(w);
    if (st != SQ_OK)
        return st;
    if (!x || !y || !ws)
        return SQ_ERR_NULL;
    if (flags & ~(SQ_ACT_STATIC_SCALE | SQ_OUT_BF16 | SQ_CHECK_FINITE))
        return SQ_ERR_ARG;
    const bool stat = (flags & SQ_ACT_STATIC_SCALE) != 0;
    if (stat && (!g_x || w->fmt != SQ_FMT_NVFP4))
        return stat && !g_x ? SQ_ERR_NULL : SQ_ERR_ARG;
    const int64_t N = w->N, K = w->K;
    if (!shape_ok_mk(M, K))
        return SQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(g_x, 4) || !aligned(ws, 256))
        return SQ_ERR_ALIGN;
    const FwdLayout L = fwd_layout(w->fmt, M, N, K);
    if (ws_bytes < L.total)
        return SQ_ERR_WORKSPACE;
    int sms = 0;
    st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool lora = w->lora_up && w->lora_down;
    uint16_t *tsplit = lora ? reinterpret_cast<uint16_t *>(ws_at(ws, L.tsplit)) : nullptr;
    uint16_t *udup = lora ? reinterpret_cast<uint16_t *>(ws_at(ws, L.udup)) : nullptr;
    float *t32 = lora ? reinterpret_cast<float *>(ws_at(ws, L.t32)) : nullptr;
    uint32_t *status = reinterpret_cast<uint32_t *>(ws_at(ws, 0));
    uint32_t *amax = reinterpret_cast<uint32_t *>(ws_at(ws, 4));
    sq::GemmLaunch g;
    memset(&g, 0, sizeof(g));
    g.M = M;
    g.N = N;
    g.K = K;
    g.y = y;
    g.out_bf16 = (flags & SQ_OUT_BF16) ? 1 : 0;
    g.status = status;
    g.tsplit = tsplit;
    g.udup = udup;
    SQ_CUDA(cudaMemsetAsync(status, 0, 8, s), "memset");   // status word + absmax
    if (w->fmt != SQ_FMT_NVFP4)       // the W ring's counters (before every kernel of the call)
        SQ_CUDA(cudaMemsetAsync(ws_at(ws, L.ring_ctr), 0, (size_t)2 * ring_slots(M, N) * 4, s), "memset");
    if (flags & SQ_CHECK_FINITE)
        SQ_CUDA(sq::launch_check_finite_bf16(x, M * K, status, sms, s), "finite check");
    if (w->fmt == SQ_FMT_NVFP4) {
        float *gx = g_x ? g_x : reinterpret_cast<float *>(ws_at(ws, 8));
        uint8_t *xc = ws_at(ws, L.a);
        uint8_t *xsf = ws_at(ws, L.a_sf);
        // one read of x for the absmax and the low-rank input, one for the quantisation
        if (!stat || lora) {
            SQ_CUDA(stage_event(SQ_STAGE_ACT_PASS1, 0, s), "event record");
            SQ_CUDA(sq::launch_act_pass1(x, M, K, w->lora_down, stat ? nullptr : amax, t32, nullptr, status, sms, s),
                    "activation pass 1");
            SQ_CUDA(stage_event(SQ_STAGE_ACT_PASS1, 1, s), "event record");
        }
        // the quantisation also writes the low-rank operands (g_x is known by then)
        sq::LowrankOut lr;
        if (lora) {
            lr.t_part = t32;
            lr.parts = sq::act_t_parts(M, K);
            lr.g_w = w->g_w;
            lr.tsplit = tsplit;
            lr.U = w->lora_up;
            lr.N = N;
            lr.udup = udup;
        }
        SQ_CUDA(stage_event(SQ_STAGE_ACT_QUANT, 0, s), "event record");
        SQ_CUDA(sq::launch_nvfp4_quant_bf16(x, M, K, amax, stat ? gx : nullptr, stat ? nullptr : gx, xc, xsf, lr,
                                            status, sms, s),
                "nvfp4 act quant + low-rank operands");
        SQ_CUDA(stage_event(SQ_STAGE_ACT_QUANT, 1, s), "event record");
        g.mode = sq::kGemmNvfp4;
        g.a = xc;
        g.b = w->codes;
        g.sfa = xsf;
        g.sfb = reinterpret_cast<const uint8_t *>(w->scales);
        g.g_x = gx;
        g.g_w = w->g_w;
    } else {
        // dequant-first: one read of x gives xb = bf16(H x) and t = x lora_down; the GEMM
        // dequantises W itself (its W ring)
        uint16_t *xb = reinterpret_cast<uint16_t *>(ws_at(ws, L.a));
        const uint16_t *Dw = w->lora_down, *Uw = w->lora_up;
        if (lora && w->fmt == SQ_FMT_INT8_ROW) {      // rank 16: zero columns 16..31
            uint16_t *d32 = reinterpret_cast<uint16_t *>(ws_at(ws, L.d32));
            uint16_t *u32 = reinterpret_cast<uint16_t *>(ws_at(ws, L.u32));
            SQ_CUDA(sq::launch_widen_rank16(w->lora_down, K, d32, sms, s), "widen lora_down");
            SQ_CUDA(sq::launch_widen_rank16(w->lora_up, N, u32, sms, s), "widen lora_up");
            Dw = d32;
            Uw = u32;
        }
        SQ_CUDA(stage_event(SQ_STAGE_ACT_PASS1, 0, s), "event record");
        SQ_CUDA(sq::launch_act_pass1(x, M, K, lora ? Dw : nullptr, nullptr, lora ? t32 : nullptr, xb, status, sms, s),
                "rotate x and low-rank input");
        SQ_CUDA(stage_event(SQ_STAGE_ACT_PASS1, 1, s), "event record");
        if (lora)
            SQ_CUDA(sq::launch_lowrank_finish(t32, sq::act_t_parts(M, K), M, nullptr, nullptr, tsplit, Uw, N, udup,
                                              sms, s),
                    "low-rank operands");
        g.mode = w->fmt == SQ_FMT_INT8_ROW ? sq::kGemmInt8
                 : w->fmt == SQ_FMT_INT4_G64 ? sq::kGemmInt4G64
                                             : sq::kGemmInt4G32;
        g.a = xb;
        g.b = w->codes;
        g.b_scales = w->scales;
        g.wring = reinterpret_cast<uint16_t *>(ws_at(ws, L.ring));
        g.ring_ctr = reinterpret_cast<uint32_t *>(ws_at(ws, L.ring_ctr));
        g.ring_slots = (int)ring_slots(M, N);
    }
    SQ_CUDA(stage_event(SQ_STAGE_GEMM, 0, s), "event record");
    SQ_CUDA(sq::launch_gemm(g, sms, s), "gemm");
    SQ_CUDA(stage_event(SQ_STAGE_GEMM, 1, s), "event record");
    return SQ_OK;
}

sq_status sq_linear_fwd_noalloc(const sq_weight *w, const uint16_t *x, int64_t M, void *y, float *g_x,
                                uint32_t flags, void **scratch_out, void *stream)
{
    static_assert(sizeof(g_noalloc_scratch) == kNoAllocScratchBytes, "scratch size");
    if (scratch_out)
        *scratch_out = nullptr;
    sq_status st = check_weight(w);
    if (st != SQ_OK)
        return st;
    if (!shape_ok_mk(M, w->K))
        return SQ_ERR_SHAPE;
    const int op = w->fmt == SQ_FMT_NVFP4      ? SQ_OP_LINEAR_FWD_NVFP4
                   : w->fmt == SQ_FMT_INT8_ROW ? SQ_OP_LINEAR_FWD_INT8
                                               : SQ_OP_LINEAR_FWD_INT4;
    const size_t need = sq_workspace_bytes(op, M, w->N, w->K);
    if (need > kNoAllocScratchBytes) {
        snprintf(g_detail, sizeof(g_detail),
                 "sq_linear_fwd_noalloc: M=%lld N=%lld K=%lld needs %zu bytes of scratch, the static scratch "
                 "holds %zu; use sq_linear_fwd with a caller workspace",
                 (long long)M, (long long)w->N, (long long)w->K, need, kNoAllocScratchBytes);
        return SQ_ERR_WORKSPACE;
    }
    int sms = 0;
    st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    int dev = 0;
    SQ_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    void *scratch = nullptr;
    {
        // first call on this device and context: look the scratch up (the device is current)
        const unsigned long long ctx = sq::current_context_id();
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        ScratchSlot &slot = g_noalloc_scratch_slot[dev];
        if (!slot.ptr || ctx == 0 || slot.ctx != ctx) {
            slot.ptr = nullptr;
            SQ_CUDA(cudaGetSymbolAddress(&slot.ptr, g_noalloc_scratch), "cudaGetSymbolAddress(static scratch)");
            slot.ctx = ctx;
        }
        scratch = slot.ptr;
    }
    if (scratch_out)
        *scratch_out = scratch;
    return sq_linear_fwd(w, x, M, y, g_x, flags, scratch, kNoAllocScratchBytes, stream);
}

sq_status sq_reconstruct_bf16(const sq_weight *w, uint16_t *W_out, uint32_t flags, void *stream)
{
    sq_status st = check_weight(w);
    if (st != SQ_OK)
        return st;
    if (!W_out)
        return SQ_ERR_NULL;
    if (flags & ~(SQ_RECON_RESIDUAL_ONLY | SQ_RECON_TRANSPOSED))
        return SQ_ERR_ARG;
    if (!aligned(W_out, 16))
        return SQ_ERR_ALIGN;
    int sms = 0;
    st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    const int with_lowrank = (!(flags & SQ_RECON_RESIDUAL_ONLY) && w->lora_up && w->lora_down) ? 1 : 0;
    const int transposed = (flags & SQ_RECON_TRANSPOSED) ? 1 : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    SQ_CUDA(sq::launch_reconstruct(w->fmt, w->codes, w->scales, w->g_w, w->lora_up, w->lora_down, w->N, w->K,
                                   with_lowrank, transposed, W_out, sms, s),
            "reconstruct");
    return SQ_OK;
}

sq_status sq_linear_bwd_dx(const sq_weight *w, const uint16_t *dy, int64_t M, float *dx, void *ws, size_t ws_bytes,
                           void *stream)
{
    sq_status st = check_weight(w);
    if (st != SQ_OK)
        return st;
    if (!dy || !dx || !ws)
        return SQ_ERR_NULL;
    const int64_t N = w->N, K = w->K;
    if (M < 1 || M > kMaxM)
        return SQ_ERR_SHAPE;
    if (!aligned(dy, 16) || !aligned(dx, 16) || !aligned(ws, 256))
        return SQ_ERR_ALIGN;
    if (ws_bytes < sq_workspace_bytes(SQ_OP_LINEAR_BWD_DX, M, N, K))
        return SQ_ERR_WORKSPACE;
    int sms = 0;
    st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws_at(ws, 0));
    uint16_t *wt = reinterpret_cast<uint16_t *>(ws_at(ws, kAlign));      // W^T [K, N] bf16
    const int with_lowrank = (w->lora_up && w->lora_down) ? 1 : 0;
    SQ_CUDA(cudaMemsetAsync(status, 0, 8, s), "memset");
    SQ_CUDA(sq::launch_reconstruct(w->fmt, w->codes, w->scales, w->g_w, w->lora_up, w->lora_down, N, K,
                                   with_lowrank, 1, wt, sms, s),
            "transposed reconstruct");
    sq::GemmLaunch g;
    memset(&g, 0, sizeof(g));
    g.mode = sq::kGemmBf16;
    g.a = dy;             // [M, N]: the reduction runs over N
    g.b = wt;             // [K, N]
    g.y = dx;             // [M, K]
    g.status = status;
    g.M = M;
    g.N = K;
    g.K = N;
    SQ_CUDA(stage_event(SQ_STAGE_GEMM, 0, s), "event record");
    SQ_CUDA(sq::launch_gemm(g, sms, s), "gemm");
    SQ_CUDA(stage_event(SQ_STAGE_GEMM, 1, s), "event record");
    return SQ_OK;
}

sq_status sq_set_stage_events(int32_t stage, void *start_event, void *stop_event)
{
    if (stage < 0 || stage >= SQ_STAGE_COUNT)
        return SQ_ERR_ARG;
    if ((start_event == nullptr) != (stop_event == nullptr))
        return SQ_ERR_NULL;
    g_stage_ev[stage][0] = reinterpret_cast<cudaEvent_t>(start_event);
    g_stage_ev[stage][1] = reinterpret_cast<cudaEvent_t>(stop_event);
    return SQ_OK;
}

sq_status sq_set_gemm_events(void *start_event, void *stop_event)
{
    return sq_set_stage_events(SQ_STAGE_GEMM, start_event, stop_event);
}

sq_status sq_selftest_wait_timeout(void *ws, uint32_t limit_us, void *stream)
{
    if (!ws)
        return SQ_ERR_NULL;
    if (!aligned(ws, 256))
        return SQ_ERR_ALIGN;
    if (limit_us < 1 || limit_us > 1000000)
        return SQ_ERR_ARG;
    int sms = 0;
    sq_status st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    SQ_CUDA(cudaMemsetAsync(status, 0, 4, s), "memset");
    selftest_wait_kernel<<<1, 32, 0, s>>>(status, 1000ull * limit_us);
    SQ_CUDA(cudaGetLastError(), "self-test launch");
    return SQ_OK;
}

sq_status sq_selftest_index_check(void *ws, void *stream)
{
    if (!ws)
        return SQ_ERR_NULL;
    if (!aligned(ws, 256))
        return SQ_ERR_ALIGN;
    int sms = 0;
    sq_status st = check_device(&sms);
    if (st != SQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    SQ_CUDA(cudaMemsetAsync(status, 0, 4, s), "memset");
    selftest_index_kernel<<<1, 32, 0, s>>>(status, 256u);
    SQ_CUDA(cudaGetLastError(), "self-test launch");
    return SQ_OK;
}

sq_status sq_check_device_status(void *ws, void *stream)
{
    if (!ws) {                                         // the library's own word (calls without a workspace)
        int sms = 0;
        sq_status st = check_device(&sms);
        if (st != SQ_OK)
            return st;
        uint32_t *word = nullptr;
        SQ_CUDA(sq::library_status_word(&word), "status symbol");
        ws = word;
    } else if (!aligned(ws, 256)) {
        return SQ_ERR_ALIGN;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    SQ_CUDA(cudaMemcpyAsync(&word, ws, 4, cudaMemcpyDeviceToHost, s), "status read");
    SQ_CUDA(cudaStreamSynchronize(s), "status sync");
    if (word != 0) {
        SQ_CUDA(cudaMemsetAsync(ws, 0, 4, s), "status clear");
        // bit 0 timeout, bit 2 failed index check, bit 1 non-finite input
        return (word & 1u) ? SQ_ERR_TIMEOUT : (word & sq::kStatusIndex) ? SQ_ERR_INDEX : SQ_ERR_NONFINITE;
    }
    return SQ_OK;
}

}  // extern "C"
