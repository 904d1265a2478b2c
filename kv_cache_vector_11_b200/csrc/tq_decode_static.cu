// Decode attention without caller-provided scratch.
//
// tq_decode_attention needs a device workspace for the per-split partial
// results (running max, running sum and unnormalised output of every context
// split).  Some callers cannot obtain one: an engine plugin whose enqueue
// path must never allocate, a serving loop that hands out device memory only
// from a fixed arena reserved at start-up, or code that must not trigger the
// implicit device-wide synchronisation cudaMalloc / cudaFree can cause in the
// middle of a decode loop.  For them this file keeps the workspace in a
// fixed-size array in the library's own device memory and passes its address
// to the unchanged decode path.  Nothing here calls cudaMalloc, cudaFree or
// any allocating library routine.

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr size_t kStaticScratchBytes = TQ_DECODE_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per device that loads the library, kept until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// cuCtxGetCurrent through the runtime's driver entry point (no link-time
// dependency on the driver library).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void * p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        cudaGetLastError();
    });
    return fn;
}

struct ScratchSlot {
    CUcontext ctx = nullptr;   // context the address was looked up in
    void * addr = nullptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices];

// Device address of g_decode_scratch in the current device's current context.
// In host code the array's name is only a host-side stand-in, so the address
// is looked up (with the device current) on the first call and cached per
// device together with the context it belongs to; a call made in another
// context -- after cudaDeviceReset tore the primary context down, or under a
// context the caller pushed -- looks it up again.
tq_status scratch_address(void ** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(TQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    }
    if (dev < 0 || dev >= kMaxDevices) return fail(TQ_ERR_UNSUPPORTED, "device ordinal >= 64");
    // (NULL before the runtime first made a context current on this thread;
    // the symbol lookup below does that)
    auto current_ctx = [] {
        CUcontext c = nullptr;
        if (CtxGetCurrentFn f = ctx_get_current())
            if (f(&c) != CUDA_SUCCESS) c = nullptr;
        return c;
    };
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot & slot = g_scratch[dev];
    if (slot.addr == nullptr || slot.ctx != current_ctx()) {
        void * p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return fail(TQ_ERR_CUDA,
                        std::string("cudaGetSymbolAddress(decode scratch): ") + cudaGetErrorString(e));
        }
        slot.addr = p;
        slot.ctx = current_ctx();
    }
    *out = slot.addr;
    return TQ_OK;
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_decode_attention_static(
    const tq_rotation * rot, int32_t k_bits, int32_t v_bits, int32_t block,
    const float * k_centroids, const float * v_centroids, const tq_rotation * qjl,
    const void * q, tq_dtype q_dtype, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
    int64_t ctx, int32_t head_dim, const uint32_t * k_codes, const uint16_t * k_norms,
    const uint32_t * qjl_signs, const uint16_t * qjl_rnorm, const uint32_t * v_codes,
    const uint16_t * v_norms, float scale, float * out, void * stream) {
    // the same plan tq_decode_attention will use for these bit widths
    int32_t qjl_m = 0;
    if (qjl != nullptr && tq_rotation_info(qjl, nullptr, &qjl_m, nullptr, nullptr) != TQ_OK) qjl_m = 0;
    const size_t need = tq::decode_need_bytes(batch, n_q_heads, n_kv_heads, ctx, head_dim, k_bits,
                                              v_bits, block == 32 ? qjl_m : -1);
    if (need > tq::kStaticScratchBytes)
        return tq::fail(TQ_ERR_UNSUPPORTED,
                        "shape needs " + std::to_string(need) +
                            " bytes of decode scratch; the built-in scratch holds " +
                            std::to_string(tq::kStaticScratchBytes) +
                            " (use tq_decode_attention with a caller workspace)");
    void * ws = nullptr;
    tq_status st = tq::scratch_address(&ws);
    if (st != TQ_OK) return st;
    // Every partial slot the combine step reads is written by the split step
    // of the same call, so the array needs no clearing between calls.
    return tq_decode_attention(rot, k_bits, v_bits, block, k_centroids, v_centroids, qjl, q,
                               q_dtype, batch, n_q_heads, n_kv_heads, ctx, head_dim, k_codes,
                               k_norms, qjl_signs, qjl_rnorm, v_codes, v_norms, scale, out, ws,
                               tq::kStaticScratchBytes, stream);
}
