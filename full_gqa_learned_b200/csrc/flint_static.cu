// flint_attn_fwd_static: the attention forward without a caller-supplied
// workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: code inside a region whose allocations are forbidden or accounted for
// elsewhere (a fixed memory budget carved out up front, an allocator that must
// not be re-entered from a callback, a plug-in host that only hands out its
// own buffers).  This entry point serves them: the scratch the kernels need
// (the work plan, the status word and the normalised FP16 keys) lives in a
// file-scope device array of fixed size, so the call itself allocates
// nothing.  Inputs and outputs are still passed by the caller.
#include <cuda_runtime.h>

#include "../../include/flint_attn.h"
#include "flint_common.cuh"

namespace flint {

flint_status_t run_stages(int stages, const void* q, const void* k, const void* v,
                          const float* q_norm_w, const float* k_norm_w, const float* sinks,
                          const int32_t* pos_ids, const int32_t* cu_seqlens, int32_t num_docs,
                          const uint8_t* pad_mask, int32_t batch, int32_t seqlen, int32_t T,
                          int32_t window, int32_t use_rope, float rope_theta, float eps, void* out,
                          float* lse, void* workspace, size_t workspace_bytes, void* stream,
                          int ng = kHKV);
flint_status_t set_error(flint_status_t s, const char* msg);

namespace {

constexpr size_t kStaticScratchBytes = FLINT_STATIC_SCRATCH_BYTES;

// Every GPU that loads the library holds this array until the process exits.
// In host code its name is only a host-side stand-in: the device address comes
// from cudaGetSymbolAddress, looked up with the device current on every call
// (cheap, allocates nothing), so no address outlives a device reset or
// belongs to another context.
__device__ __align__(256) char g_scratch[kStaticScratchBytes];

flint_status_t scratch_address(void** addr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p)
        return set_error(FLINT_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
    *addr = p;
    return FLINT_OK;
}

}  // namespace
}  // namespace flint

extern "C" {

flint_status_t flint_attn_fwd_static(const void* q, const void* k, const void* v,
                                     const float* q_norm_w, const float* k_norm_w,
                                     const float* sinks, const int32_t* pos_ids,
                                     const int32_t* cu_seqlens, int32_t num_docs,
                                     const uint8_t* pad_mask, int32_t batch, int32_t seqlen,
                                     int32_t T, int32_t window, int32_t use_rope,
                                     float rope_theta, float eps, void* out, float* lse,
                                     void* stream) {
    int32_t nseg = 1;
    if (cu_seqlens) nseg = num_docs;
    else if (pad_mask) nseg = batch;
    const size_t need = flint_attn_workspace_bytes(T, nseg < 0 ? 0 : nseg);
    if (T > 0 && (need == 0 || need > flint::kStaticScratchBytes))
        return flint::set_error(FLINT_ERR_WORKSPACE,
                                "problem needs more scratch than the static array holds; "
                                "use flint_attn_fwd with a workspace");
    void* scratch = nullptr;
    if (T > 0) {
        const flint_status_t st = flint::scratch_address(&scratch);
        if (st != FLINT_OK) return st;
    }
    return flint::run_stages(flint::kStageBoth, q, k, v, q_norm_w, k_norm_w, sinks, pos_ids,
                             cu_seqlens, num_docs, pad_mask, batch, seqlen, T, window, use_rope,
                             rope_theta, eps, out, lse, scratch, flint::kStaticScratchBytes,
                             stream);
}

flint_status_t flint_attn_fwd_static_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return flint::set_error(FLINT_ERR_CUDA, "stream synchronisation failed");
    // the status word is the first word of the work-plan header, which sits
    // at the start of the scratch
    int st = 0;
    e = cudaMemcpyFromSymbol(&st, flint::g_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess)
        return flint::set_error(FLINT_ERR_CUDA, "reading the static scratch's status failed");
    return static_cast<flint_status_t>(st);
}

}  // extern "C"
