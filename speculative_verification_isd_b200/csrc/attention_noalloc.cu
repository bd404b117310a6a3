// isd_attention_noalloc: the attention step (KV append + paged GQA attention)
// for callers that cannot give the library a workspace.
//
// Who needs it: a serving engine that hands all free device memory to its KV
// cache pool when it starts (so nothing is left to allocate per step), and
// code that must not call the CUDA allocator at all, for instance because
// cudaMalloc/cudaFree may synchronise the device in the middle of a pipelined
// decode loop.  Such callers still pass every input and output buffer; only
// the scratch that the split-KV attention needs (per-split partial results
// and the last-CTA counters) comes from a fixed array inside the library.
//
// That array is a file-scope __device__ array of kNoAllocScratchBytes bytes.
// Every GPU that loads the library keeps it for the life of the process.  All
// calls on a device share it: two calls that overlap on the GPU (different
// streams, no ordering between them) race on it.  Its counters are cleared on
// the caller's stream at every call; the partial results need no clearing.
//
// Host code cannot use the array's name as a device address, so the first
// call on each device (with that device current) looks the address up with
// cudaGetSymbolAddress and keeps it, together with the unique id of the
// context it was looked up in; a later call in another context on the same
// device (after cudaDeviceReset, for instance) looks it up again.  Make the
// first call on a device, and the first one after a reset, before any stream
// capture.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "plan.h"

#define ISD_NOALLOC_MAX_DEVICES 64

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)ISD_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_attn_scratch[kNoAllocScratchBytes];

struct ScratchSlot {
    void* ptr;             // device address of g_attn_scratch in that context
    unsigned long long ctx_id;  // unique id of the context of the lookup
};
ScratchSlot g_scratch[ISD_NOALLOC_MAX_DEVICES];  // per device, filled on first use
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if there is none yet
// or the driver cannot say).
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked = false;
    if (!looked) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        looked = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_cur && get_id && get_cur(&ctx) == CUDA_SUCCESS && ctx &&
        get_id(ctx, &id) == CUDA_SUCCESS)
        return id;
    return 0;
}

}  // namespace

namespace isd {
cudaError_t launch_attention(const Plan& p, const isd_dims* d, const uint16_t* q,
                             const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_pool,
                             uint16_t* v_pool, const int32_t* page_table, const int32_t* kv_len,
                             const int32_t* n_clean, uint16_t* out, void* ws, int32_t* err_flag,
                             cudaStream_t st, int* clear_extra, int* clear_range, int clear_count,
                             bool pdl, bool bidir);
void set_last_error(const char* msg);
}  // namespace isd

extern "C" isd_status isd_attention_noalloc(const isd_dims* d, const uint16_t* q,
                                            const uint16_t* k_new, const uint16_t* v_new,
                                            uint16_t* k_pool, uint16_t* v_pool,
                                            const int32_t* page_table, const int32_t* kv_len,
                                            const int32_t* n_clean, uint16_t* out,
                                            int32_t* err_flag, void* stream) {
    isd::Plan p;
    if (!isd::make_plan(d, &p)) {
        isd::set_last_error("isd_attention_noalloc: invalid dims");
        return ISD_ERR_INVALID_ARG;
    }
    if (!q || !k_new || !v_new || !k_pool || !v_pool || !page_table || !kv_len || !n_clean ||
        !out) {
        isd::set_last_error("isd_attention_noalloc: null pointer");
        return ISD_ERR_INVALID_ARG;
    }
    if ((d->D != 64 && d->D != 128) || p.rows > 128) {
        isd::set_last_error("isd_attention_noalloc: unsupported head dim or block rows");
        return ISD_ERR_UNSUPPORTED_SHAPE;
    }
    // The attention uses the workspace from offset 0 up to the end of its
    // counters (off_hidden): that much must fit in the built-in array.
    const size_t need = p.off_hidden;
    if (need > kNoAllocScratchBytes) {
        char msg[160];
        snprintf(msg, sizeof(msg),
                 "isd_attention_noalloc: needs %zu bytes of scratch, more than the built-in %zu",
                 need, kNoAllocScratchBytes);
        isd::set_last_error(msg);
        return ISD_ERR_WORKSPACE;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= ISD_NOALLOC_MAX_DEVICES) {
        isd::set_last_error("isd_attention_noalloc: no usable current device");
        return ISD_ERR_CUDA;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        ScratchSlot& slot = g_scratch[dev];
        const unsigned long long id = current_ctx_id();
        if (!slot.ptr || id == 0 || id != slot.ctx_id) {
            void* ptr = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&ptr, g_attn_scratch);
            if (e != cudaSuccess || !ptr) {
                isd::set_last_error("isd_attention_noalloc: device address of the scratch array");
                return ISD_ERR_CUDA;
            }
            slot.ptr = ptr;
            // the lookup has made the context current if it was not yet
            slot.ctx_id = current_ctx_id();
        }
        scratch = slot.ptr;
    }
    char* ws = static_cast<char*>(scratch);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // launch_attention clears the counters on the stream before the attention
    if (isd::launch_attention(p, d, q, k_new, v_new, k_pool, v_pool, page_table, kv_len, n_clean,
                              out, ws, err_flag, st, nullptr, nullptr, 0, false, false) != cudaSuccess) {
        isd::set_last_error("isd_attention_noalloc: launch failed");
        return ISD_ERR_CUDA;
    }
    return ISD_OK;
}
