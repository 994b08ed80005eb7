// lisa_topm_noalloc: the indexer-score + top-M selection of lisa_topm for
// callers that cannot hand the library a workspace.
//
// Some callers have no way to allocate device memory for the library: code
// that runs inside a host framework whose device allocator it may not touch,
// plugin or callback interfaces that only pass in the tensors of the call, and
// latency-critical loops where a cudaMalloc (which can synchronise the device)
// is not acceptable.  This entry point needs nothing beyond the inputs and
// outputs: the per-call scores live in a fixed device array that is part of the
// library image.
//
// Costs and rules of that array:
//  - it holds kScratchBytes (4 MiB) on every GPU that loads the library, until
//    the process exits;
//  - a call whose scores need more than that (B * T * (n_past + T) floats) is
//    rejected with LISA_ERR_UNSUPPORTED before anything is launched;
//  - every call on a device shares it and it keeps the last call's contents
//    (each call writes every score it later reads, so nothing needs clearing);
//    calls that may overlap on the GPU (different streams without ordering, or
//    several host threads) race on it and must be serialised by the caller;
//  - the first call on each device looks up the array's device address (a
//    one-time set-up with that device current); make that first call before
//    any stream capture begins.  The address belongs to the device's current
//    context: after cudaDeviceReset the next call sees a new context and looks
//    the address up again (that call, too, must come before any capture).
#include <cuda.h>

#include <mutex>

#include "lisa_internal.cuh"

namespace lisa {
namespace {

constexpr size_t kScratchBytes = 4u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Process-unique id of the current context (0 when the driver cannot say):
// a reset device gets a new context, and with it a new id.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    }
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array on the current device (nullptr on
// failure).  In host code the array's name is only a host-side stand-in, so the
// address must come from cudaGetSymbolAddress with the device current; it is
// looked up once per device and context.
void* scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_addr[dev] || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    return g_scratch_addr[dev];
}

}  // namespace
}  // namespace lisa

extern "C" LISA_API lisa_status lisa_topm_noalloc(const lisa_dims* dims, const void* q_I,
                                                  const void* k_I_cache, const float* w,
                                                  int64_t w_tok_stride, int32_t* idx,
                                                  int32_t* count, void* stream) {
    using namespace lisa;
    size_t probe = 0;
    const lisa_status st = lisa_workspace_size(dims, LISA_OP_TOPM, &probe);  // validates dims
    if (st != LISA_OK) return st;
    if (!(w_tok_stride == 0 || w_tok_stride == dims->H_I)) return LISA_ERR_INVALID_ARG;
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!q_I || !k_I_cache || !w || !idx || !count) return LISA_ERR_INVALID_ARG;
    const size_t need = sizeof(float) * (size_t)s.B * s.T * s.L;
    if (need > kScratchBytes) return LISA_ERR_UNSUPPORTED;
    float* scores = static_cast<float*>(scratch_for_current_device());
    if (!scores) return LISA_ERR_CUDA;
    cudaStream_t cs = (cudaStream_t)stream;
    if (generic_index_scores(s, q_I, k_I_cache, w, w_tok_stride, scores, cs) != cudaSuccess)
        return LISA_ERR_CUDA;
    if (generic_topm_from_scores(s, scores, idx, count, cs) != cudaSuccess) return LISA_ERR_CUDA;
    return LISA_OK;
}
