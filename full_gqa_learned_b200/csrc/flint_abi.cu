// Host side of the C ABI declared in include/flint_attn.h: argument
// validation, workspace layout, TMA tensor maps and the two launches
// (preparation kernel, attention kernel).  No allocation, no host<->device
// copies, no synchronisation on the call path.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>

#include <nvtx3/nvToolsExt.h>   // header-only NVTX v3: named ranges for profilers
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/flint_attn.h"
#include "flint_common.cuh"
#include "flint_host.cuh"

namespace flint {
template <bool kSplit>
__global__ void prep_kernel(PrepParams p);
__global__ void attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                                const __grid_constant__ CUtensorMap tm_k,
                                const __grid_constant__ CUtensorMap tm_v,
                                const __grid_constant__ CUtensorMap tm_o,
                                const __grid_constant__ CUtensorMap tm_o1, const AttnParams p);
__global__ void attn_fwd_qprep_kernel(const __grid_constant__ CUtensorMap tm_q,
                                      const __grid_constant__ CUtensorMap tm_k,
                                      const __grid_constant__ CUtensorMap tm_v,
                                      const __grid_constant__ CUtensorMap tm_o,
                                      const __grid_constant__ CUtensorMap tm_o1, const AttnParams p);
__global__ void attn_fwd_f16_kernel(const __grid_constant__ CUtensorMap tm_q,
                                    const __grid_constant__ CUtensorMap tm_k,
                                    const __grid_constant__ CUtensorMap tm_v,
                                    const __grid_constant__ CUtensorMap tm_o,
                                    const __grid_constant__ CUtensorMap tm_o1, const AttnParams p);
extern const unsigned kAttnSmemBytes;
extern const unsigned kAttnThreads;
}  // namespace flint

using namespace flint;

namespace {
thread_local char g_err[512] = "";
std::mutex g_mu;
}  // namespace

namespace flint {

flint_status_t fail(flint_status_t s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

namespace {
EncodeTiledFn g_encode = nullptr;
constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
bool g_attr_set[kMaxDevices] = {false};
}  // namespace

flint_status_t get_encoder(EncodeTiledFn* fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled unavailable: %s",
                        cudaGetErrorString(e));
        g_encode = reinterpret_cast<EncodeTiledFn>(p);
    }
    *fn = g_encode;
    return FLINT_OK;
}

flint_status_t device_setup(int* sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(FLINT_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_attr_set[dev]) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0)
            return fail(FLINT_ERR_UNSUPPORTED, "needs an sm_100 GPU, found sm_%d%d", major, minor);
        e = cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kAttnSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(attn_fwd_f16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kAttnSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(attn_fwd_qprep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kAttnSmemBytes);
        if (e != cudaSuccess)
            return fail(FLINT_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev);
        g_attr_set[dev] = true;
    }
    *sms = g_sms[dev];
    return FLINT_OK;
}

}  // namespace flint

namespace {

// 3-D map over a [T, heads, 128] tensor of 16-bit elements: dims (128, heads,
// T), box (64, box_heads, box_tokens), 128-byte swizzle, zero fill outside.
flint_status_t make_map(EncodeTiledFn enc, CUtensorMap* m, CUtensorMapDataType dt, const void* base,
                        int heads, int T, int box_heads, int box_tokens) {
    cuuint64_t dims[3] = {(cuuint64_t)kHD, (cuuint64_t)heads, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)kHD * 2, (cuuint64_t)heads * kHD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return FLINT_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Test hook, not part of the ABI.  FLINT_TEST_WAIT_TIMEOUT_MS=n (1..10000),
// read once when the process first launches the attention kernel, makes that
// one launch's MMA warps wait n ms on a barrier nothing arrives on, so the
// bounded-wait timeout path runs; later launches are unaffected.
std::once_flag g_stall_once;
std::atomic<unsigned long long> g_stall_ns{0};

unsigned long long test_stall_once() {
    std::call_once(g_stall_once, [] {
        if (const char* tw = std::getenv("FLINT_TEST_WAIT_TIMEOUT_MS")) {
            const long ms = std::strtol(tw, nullptr, 10);
            if (ms > 0 && ms <= 10000) g_stall_ns.store((unsigned long long)ms * 1000000ull);
        }
    });
    if (g_stall_ns.load(std::memory_order_relaxed) == 0) return 0;
    return g_stall_ns.exchange(0);
}

}  // namespace

extern "C" {

int32_t flint_attn_abi_version(void) { return 1; }

size_t flint_attn_workspace_bytes(int32_t T, int32_t num_segments) {
    if (T < 0 || T > FLINT_MAX_TOKENS || num_segments < 0 || num_segments > FLINT_MAX_TOKENS)
        return 0;
    int nseg = num_segments < 1 ? 1 : num_segments;
    return ws_layout(T, nseg).total;
}

const char* flint_attn_last_error(void) { return g_err; }

const char* flint_attn_status_string(flint_status_t s) {
    switch (s) {
        case FLINT_OK: return "FLINT_OK";
        case FLINT_ERR_INVALID_ARG: return "FLINT_ERR_INVALID_ARG";
        case FLINT_ERR_UNSUPPORTED: return "FLINT_ERR_UNSUPPORTED";
        case FLINT_ERR_CUDA: return "FLINT_ERR_CUDA";
        case FLINT_ERR_TIMEOUT: return "FLINT_ERR_TIMEOUT";
        case FLINT_ERR_WORKSPACE: return "FLINT_ERR_WORKSPACE";
    }
    return "FLINT_ERR_UNKNOWN";
}

}  // extern "C"

namespace flint {

flint_status_t run_stages(int stages, const void* q, const void* k, const void* v, const float* q_norm_w,
                   const float* k_norm_w, const float* sinks, const int32_t* pos_ids,
                   const int32_t* cu_seqlens, int32_t num_docs, const uint8_t* pad_mask,
                   int32_t batch, int32_t seqlen, int32_t T, int32_t window, int32_t use_rope,
                   float rope_theta, float eps, void* out, float* lse, void* workspace,
                   size_t workspace_bytes, void* stream, int ng = kHKV) {
    g_err[0] = '\0';
    if (ng != 1 && ng != 2 && ng != 4)
        return fail(FLINT_ERR_INVALID_ARG, "kv_heads=%d: a head slice has 1, 2 or 4 KV heads", ng);
    if (ng != kHKV && (stages & (kStageF16 | kStageKeysReady)))
        return fail(FLINT_ERR_UNSUPPORTED, "head slices use the BF16 forward only");
    // ---- host-side validation: nothing below touches the GPU until it passes
    if (T < 0 || T > FLINT_MAX_TOKENS)
        return fail(FLINT_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, FLINT_MAX_TOKENS);
    if (window < 0) return fail(FLINT_ERR_INVALID_ARG, "window=%d < 0", window);
    if (use_rope != 0 && use_rope != 1) return fail(FLINT_ERR_INVALID_ARG, "use_rope must be 0 or 1");
    if (!(eps > 0.f) || !std::isfinite(eps)) return fail(FLINT_ERR_INVALID_ARG, "eps must be > 0");
    if (use_rope && (!(rope_theta > 1.f) || !std::isfinite(rope_theta)))
        return fail(FLINT_ERR_INVALID_ARG, "rope_theta must be > 1");
    if (cu_seqlens && pad_mask)
        return fail(FLINT_ERR_INVALID_ARG, "give at most one of cu_seqlens and pad_mask");
    int mode = kMaskSingle, nseg = 1;
    if (cu_seqlens) {
        if (num_docs < 0 || num_docs > FLINT_MAX_TOKENS)
            return fail(FLINT_ERR_INVALID_ARG, "num_docs=%d", num_docs);
        mode = kMaskThd;
        nseg = num_docs;
    } else if (pad_mask) {
        if (batch < 1 || seqlen < 1 || (long long)batch * seqlen != (long long)T)
            return fail(FLINT_ERR_INVALID_ARG, "pad_mask needs batch*seqlen == T (%d*%d vs %d)",
                        batch, seqlen, T);
        mode = kMaskPad;
        nseg = batch;
    }
    if (T == 0) return FLINT_OK;
    if (!q || !k || !v || !q_norm_w || !k_norm_w || !sinks || !out)
        return fail(FLINT_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return fail(FLINT_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
    if (!aligned(q_norm_w, 4) || !aligned(k_norm_w, 4) || !aligned(sinks, 4) ||
        (lse && !aligned(lse, 4)) || (pos_ids && !aligned(pos_ids, 4)) ||
        (cu_seqlens && !aligned(cu_seqlens, 4)))
        return fail(FLINT_ERR_INVALID_ARG, "misaligned 32-bit array");
    const bool f16 = (stages & kStageF16) != 0;
    // Queries: prepared on tile load by the attention kernel on full layers;
    // on sliding layers (short units, measured faster) by the preparation
    // kernel into the output rows, unless the caller asks for tile load
    const bool qprep = !f16 && window > 0 && !(stages & kStageTileQ);
    const WsLayout L = ws_layout(T, nseg < 1 ? 1 : nseg);
    const size_t need = f16 ? L.total_f16 : L.total;
    if (!workspace || !aligned(workspace, 256))
        return fail(FLINT_ERR_WORKSPACE, "workspace missing or not 256-byte aligned");
    if (workspace_bytes < need)
        return fail(FLINT_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);

    // ---- launch
    int sms = 0;
    flint_status_t st = device_setup(&sms);
    if (st != FLINT_OK) return st;
    EncodeTiledFn enc = nullptr;
    st = get_encoder(&enc);
    if (st != FLINT_OK) return st;
    char* ws = static_cast<char*>(workspace);
    CUtensorMap tm_q, tm_k, tm_v, tm_o, tm_o1;
    // Q tiles: the raw BF16 queries, normalised and rotated in shared memory
    // by the attention kernel (FP16 policy: the FP16 queries the preparation
    // kernel normalised and rotated into the workspace)
    const CUtensorMapDataType t16 = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int nh = kGroup * ng;      // query heads in the tensors
    if (f16)
        st = make_map(enc, &tm_q, t16, ws + L.qn, nh, T, kGroup, kTokPerTile);
    else if (qprep)
        st = make_map(enc, &tm_q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, out, nh, T, kGroup, kTokPerTile);
    else
        st = make_map(enc, &tm_q, t16, q, nh, T, kGroup, kTokPerTile);
    if (st != FLINT_OK) return st;
    st = make_map(enc, &tm_k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + L.kn, ng, T, 1, kKeyChunk);
    if (st != FLINT_OK) return st;
    // result: 4 tokens (the rows of one softmax warp), and single tokens
    // where a document ends inside a warp's 4
    st = make_map(enc, &tm_o, t16, out, nh, T, kGroup, 4);
    if (st != FLINT_OK) return st;
    st = make_map(enc, &tm_o1, t16, out, nh, T, kGroup, 1);
    if (st != FLINT_OK) return st;
    st = make_map(enc, &tm_v, t16, f16 ? static_cast<const void*>(ws + L.vh) : v, ng, T, 1, kKeyChunk);
    if (st != FLINT_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    PrepParams pp;
    pp.q = static_cast<const __nv_bfloat16*>(q);
    pp.k = static_cast<const __nv_bfloat16*>(k);
    pp.q_norm_w = q_norm_w;
    pp.k_norm_w = k_norm_w;
    pp.sinks = sinks;
    pp.pos_ids = pos_ids;
    pp.cu_seqlens = cu_seqlens;
    pp.pad_mask = pad_mask;
    pp.out = static_cast<__nv_bfloat16*>(out);
    pp.lse = lse;
    pp.ws = ws;
    pp.T = T;
    pp.nseg = nseg < 1 ? (mode == kMaskThd ? 0 : 1) : nseg;
    pp.batch = batch;
    pp.seqlen = seqlen;
    pp.window = window;
    pp.use_rope = use_rope;
    pp.mode = mode;
    pp.keys_ready = (stages & kStageKeysReady) ? 1 : 0;
    pp.ng = ng;
    pp.qprep = qprep ? 1 : 0;
    pp.f16 = f16 ? 1 : 0;
    pp.qf = f16 ? static_cast<const float*>(q) : nullptr;
    pp.kf = f16 ? static_cast<const float*>(k) : nullptr;
    pp.vf = f16 ? static_cast<const float*>(v) : nullptr;
    if (f16) {
        pp.q = nullptr;
        pp.k = nullptr;
    }
    pp.rope_theta = rope_theta;
    pp.eps = eps;
    // ws_layout is always evaluated with max(nseg, 1) segments
    // block 0 plans; the others take warps' worth of token work, at most
    // four blocks per SM (they loop over the rest)
    const int prep_n = prep_parts(T, f16 || qprep);
    const bool prep_split = prep_n > 1;
    long long prep_blocks_ll = 1 + ((long long)T * prep_n + 31) / 32;
    if (prep_blocks_ll > 1 + 4LL * sms) prep_blocks_ll = 1 + 4LL * sms;
    int prep_blocks = (int)prep_blocks_ll;
    if (prep_blocks < 2) prep_blocks = 2;
    if (stages & kStagePrepare) {
        if (prep_split)
            prep_kernel<true><<<prep_blocks, 1024, 0, s>>>(pp);
        else
            prep_kernel<false><<<prep_blocks, 1024, 0, s>>>(pp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "prep launch: %s", cudaGetErrorString(e));
    }
    if (!(stages & kStageAttend)) return FLINT_OK;

    AttnParams ap;
    ap.q_norm_w = q_norm_w;
    ap.k_norm_w = k_norm_w;
    ap.sinks = sinks;
    ap.pos_ids = pos_ids;
    ap.out = static_cast<__nv_bfloat16*>(out);
    ap.lse = lse;
    ap.ws = ws;
    ap.T = T;
    ap.nseg = pp.nseg;
    ap.window = window;
    ap.use_rope = use_rope;
    ap.ng = ng;
    ap.rope_theta = rope_theta;
    ap.eps = eps;
    ap.test_wait_ns = test_stall_once();
    const int max_units = L.max_items * ng;
    const int grid = max_units < sms ? max_units : sms;
    if (stages & kStagePrepare) {
        // launched right behind the preparation kernel: a programmatic
        // dependent, so its setup overlaps the preparation kernel's tail
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kAttnThreads);
        cfg.dynamicSmemBytes = kAttnSmemBytes;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = f16     ? cudaLaunchKernelEx(&cfg, attn_fwd_f16_kernel, tm_q, tm_k, tm_v, tm_o, tm_o1, ap)
            : qprep ? cudaLaunchKernelEx(&cfg, attn_fwd_qprep_kernel, tm_q, tm_k, tm_v, tm_o, tm_o1, ap)
                    : cudaLaunchKernelEx(&cfg, attn_fwd_kernel, tm_q, tm_k, tm_v, tm_o, tm_o1, ap);
    } else {
        if (f16)
            attn_fwd_f16_kernel<<<grid, kAttnThreads, kAttnSmemBytes, s>>>(tm_q, tm_k, tm_v, tm_o, tm_o1, ap);
        else if (qprep)
            attn_fwd_qprep_kernel<<<grid, kAttnThreads, kAttnSmemBytes, s>>>(tm_q, tm_k, tm_v, tm_o, tm_o1, ap);
        else
            attn_fwd_kernel<<<grid, kAttnThreads, kAttnSmemBytes, s>>>(tm_q, tm_k, tm_v, tm_o, tm_o1, ap);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
    return FLINT_OK;
}

flint_status_t set_error(flint_status_t s, const char* msg) { return fail(s, "%s", msg); }

struct GemmParams;
flint_status_t launch_qkv_gemm(const void* x, const void* w_qkv, int T, int hidden, void* q, void* k,
                               void* v, void* kn, const float* k_norm_w, float eps, int use_rope,
                               float rope_theta, const int32_t* pos_ids, const int32_t* cu_seqlens,
                               int nseg, int seqlen, int* status, cudaStream_t s);
flint_status_t launch_plain_gemm(const void* a, const void* b, int M, int N, int K, void* c, int* status,
                                 cudaStream_t s);

size_t decode_workspace_bytes(int B, int cap, int window);
flint_status_t run_decode(const void* q, const void* k, const void* v, const float* q_norm_w,
                          const float* k_norm_w, const float* sinks, void* k_cache, void* v_cache,
                          const int32_t* cache_len, int32_t B, int32_t cap, int32_t window,
                          int32_t use_rope, float rope_theta, float eps, void* out, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream);

size_t bwd_workspace_bytes(int T);
flint_status_t run_bwd(const void* q, const void* k, const void* v, const float* q_norm_w,
                       const float* k_norm_w, const float* sinks, const int32_t* pos_ids,
                       const int32_t* cu_seqlens, int32_t num_docs, const uint8_t* pad_mask,
                       int32_t batch, int32_t seqlen, int32_t T, int32_t window, int32_t use_rope,
                       float rope_theta, float eps, const void* out, const float* lse, const void* dout,
                       float* dq, float* dk, float* dv, float* dq_norm_w, float* dk_norm_w,
                       float* dsinks, void* workspace, int sms, void* stream);

}  // namespace flint

extern "C" {

#define FLINT_ARGS                                                                            \
    const void *q, const void *k, const void *v, const float *q_norm_w, const float *k_norm_w, \
        const float *sinks, const int32_t *pos_ids, const int32_t *cu_seqlens, int32_t num_docs, \
        const uint8_t *pad_mask, int32_t batch, int32_t seqlen, int32_t T, int32_t window,       \
        int32_t use_rope, float rope_theta, float eps, void *out, float *lse, void *workspace,   \
        size_t workspace_bytes, void *stream
#define FLINT_FWD_ARGS                                                                         \
    q, k, v, q_norm_w, k_norm_w, sinks, pos_ids, cu_seqlens, num_docs, pad_mask, batch, seqlen, \
        T, window, use_rope, rope_theta, eps, out, lse, workspace, workspace_bytes, stream

// Each entry point is one NVTX range (host side: the enqueue), so a timeline
// profiler shows which library call launched which kernels.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

flint_status_t flint_attn_fwd(FLINT_ARGS) {
    NvtxRange r("flint_attn_fwd");
    return run_stages(kStageBoth, FLINT_FWD_ARGS);
}
flint_status_t flint_attn_fwd_heads(const void* q, const void* k, const void* v, const float* q_norm_w,
                                    const float* k_norm_w, const float* sinks, const int32_t* pos_ids,
                                    const int32_t* cu_seqlens, int32_t num_docs, const uint8_t* pad_mask,
                                    int32_t batch, int32_t seqlen, int32_t T, int32_t kv_heads,
                                    int32_t window, int32_t use_rope, float rope_theta, float eps, void* out,
                                    float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange r("flint_attn_fwd_heads");
    return run_stages(kStageBoth, FLINT_FWD_ARGS, kv_heads);
}
size_t flint_attn_fp16_workspace_bytes(int32_t T, int32_t num_segments) {
    if (T < 0 || T > FLINT_MAX_TOKENS || num_segments < 0 || num_segments > FLINT_MAX_TOKENS)
        return 0;
    return ws_layout(T, num_segments < 1 ? 1 : num_segments).total_f16;
}
flint_status_t flint_attn_fwd_fp16(const float* q, const float* k, const float* v, const float* q_norm_w,
                                   const float* k_norm_w, const float* sinks, const int32_t* pos_ids,
                                   const int32_t* cu_seqlens, int32_t num_docs, const uint8_t* pad_mask,
                                   int32_t batch, int32_t seqlen, int32_t T, int32_t window,
                                   int32_t use_rope, float rope_theta, float eps, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange r("flint_attn_fwd_fp16");
    return run_stages(kStageBoth | kStageF16, FLINT_FWD_ARGS);
}
flint_status_t flint_attn_prepare(FLINT_ARGS) {
    NvtxRange r("flint_attn_prepare");
    return run_stages(kStagePrepare, FLINT_FWD_ARGS);
}
flint_status_t flint_attn_attend(FLINT_ARGS) {
    NvtxRange r("flint_attn_attend");
    return run_stages(kStageAttend, FLINT_FWD_ARGS);
}

namespace {

flint_status_t check_proj(int32_t T, int32_t hidden) {
    if (T < 0 || T > FLINT_MAX_TOKENS)
        return fail(FLINT_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, FLINT_MAX_TOKENS);
    if (hidden < 64 || hidden > FLINT_MAX_HIDDEN || hidden % 64 != 0)
        return fail(FLINT_ERR_INVALID_ARG, "hidden=%d must be a multiple of 64 in [64, %d]", hidden,
                    FLINT_MAX_HIDDEN);
    return FLINT_OK;
}

}  // namespace

flint_status_t flint_qkv_proj(const void* x, const void* w_qkv, int32_t T, int32_t hidden, void* q,
                              void* k, void* v, void* stream) {
    NvtxRange r("flint_qkv_proj");
    g_err[0] = '\0';
    flint_status_t st = check_proj(T, hidden);
    if (st != FLINT_OK) return st;
    if (T == 0) return FLINT_OK;
    if (!x || !w_qkv || !q || !k || !v) return fail(FLINT_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16))
        return fail(FLINT_ERR_INVALID_ARG, "x, w_qkv, q, k and v must be 16-byte aligned");
    return flint::launch_qkv_gemm(x, w_qkv, T, hidden, q, k, v, nullptr, nullptr, 1e-6f, 0, 10000.f,
                                  nullptr, nullptr, 0, 0, nullptr, static_cast<cudaStream_t>(stream));
}

flint_status_t flint_o_proj(const void* attn_out, const void* w_o, int32_t T, int32_t hidden, void* y,
                            void* stream) {
    NvtxRange r("flint_o_proj");
    g_err[0] = '\0';
    flint_status_t st = check_proj(T, hidden);
    if (st != FLINT_OK) return st;
    if (T == 0) return FLINT_OK;
    if (!attn_out || !w_o || !y) return fail(FLINT_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(attn_out, 16) || !aligned(w_o, 16) || !aligned(y, 16))
        return fail(FLINT_ERR_INVALID_ARG, "attn_out, w_o and y must be 16-byte aligned");
    return flint::launch_plain_gemm(attn_out, w_o, T, hidden, kHQ * kHD, y, nullptr,
                                    static_cast<cudaStream_t>(stream));
}

flint_status_t flint_attn_layer_fwd(const void* x, const void* w_qkv, const void* w_o,
                                    const float* q_norm_w, const float* k_norm_w, const float* sinks,
                                    const int32_t* pos_ids, const int32_t* cu_seqlens, int32_t num_docs,
                                    const uint8_t* pad_mask, int32_t batch, int32_t seqlen, int32_t T,
                                    int32_t hidden, int32_t window, int32_t use_rope, float rope_theta,
                                    float eps, void* q, void* k, void* v, void* attn_out, void* y,
                                    float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange r("flint_attn_layer_fwd");
    g_err[0] = '\0';
    flint_status_t st = check_proj(T, hidden);
    if (st != FLINT_OK) return st;
    if (T > 0) {
        if (!x || !w_qkv || !w_o || !y) return fail(FLINT_ERR_INVALID_ARG, "null tensor pointer");
        if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(w_o, 16) || !aligned(y, 16))
            return fail(FLINT_ERR_INVALID_ARG, "x, w_qkv, w_o and y must be 16-byte aligned");
    }
    // 1. plan and padded rows (every other argument is validated here, before
    //    any launch); the keys come from the projection's epilogue
    st = run_stages(kStagePrepare | kStageKeysReady | kStageTileQ, q, k, v, q_norm_w, k_norm_w, sinks, pos_ids,
                    cu_seqlens, num_docs, pad_mask, batch, seqlen, T, window, use_rope, rope_theta, eps,
                    attn_out, lse, workspace, workspace_bytes, stream);
    if (st != FLINT_OK || T == 0) return st;
    int nseg = 1;
    if (cu_seqlens) nseg = num_docs;
    else if (pad_mask) nseg = batch;
    const WsLayout L = ws_layout(T, nseg < 1 ? 1 : nseg);
    char* ws = static_cast<char*>(workspace);
    int* status = &reinterpret_cast<PlanHeader*>(ws + L.header)->status;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // 2. q, k, v and the attention kernel's key operand
    st = flint::launch_qkv_gemm(x, w_qkv, T, hidden, q, k, v, ws + L.kn, k_norm_w, eps, use_rope, rope_theta,
                                pos_ids, cu_seqlens, cu_seqlens ? num_docs : 0, pad_mask ? seqlen : 0,
                                status, s);
    if (st != FLINT_OK) return st;
    // 3. attention
    st = run_stages(kStageAttend | kStageTileQ, q, k, v, q_norm_w, k_norm_w, sinks, pos_ids, cu_seqlens, num_docs,
                    pad_mask, batch, seqlen, T, window, use_rope, rope_theta, eps, attn_out, lse, workspace,
                    workspace_bytes, stream);
    if (st != FLINT_OK) return st;
    // 4. o_proj
    return flint::launch_plain_gemm(attn_out, w_o, T, hidden, kHQ * kHD, y, status, s);
}

size_t flint_attn_decode_workspace_bytes(int32_t B, int32_t cap, int32_t window) {
    if (B < 0 || B > FLINT_MAX_DECODE_BATCH || cap < 1 || cap > FLINT_MAX_TOKENS || window < 0) return 0;
    return flint::decode_workspace_bytes(B, cap, window);
}

flint_status_t flint_attn_decode(const void* q, const void* k, const void* v, const float* q_norm_w,
                                 const float* k_norm_w, const float* sinks, void* k_cache,
                                 void* v_cache, const int32_t* cache_len, int32_t B, int32_t cap,
                                 int32_t window, int32_t use_rope, float rope_theta, float eps,
                                 void* out, float* lse, void* workspace, size_t workspace_bytes,
                                 void* stream) {
    NvtxRange r("flint_attn_decode");
    g_err[0] = '\0';
    if (B < 0 || B > FLINT_MAX_DECODE_BATCH)
        return fail(FLINT_ERR_INVALID_ARG, "B=%d outside [0, %d]", B, FLINT_MAX_DECODE_BATCH);
    if (cap < 1 || cap > FLINT_MAX_TOKENS) return fail(FLINT_ERR_INVALID_ARG, "cap=%d", cap);
    if (window < 0) return fail(FLINT_ERR_INVALID_ARG, "window=%d < 0", window);
    if (use_rope != 0 && use_rope != 1) return fail(FLINT_ERR_INVALID_ARG, "use_rope must be 0 or 1");
    if (!(eps > 0.f) || !std::isfinite(eps)) return fail(FLINT_ERR_INVALID_ARG, "eps must be > 0");
    if (use_rope && (!(rope_theta > 1.f) || !std::isfinite(rope_theta)))
        return fail(FLINT_ERR_INVALID_ARG, "rope_theta must be > 1");
    if (B == 0) return FLINT_OK;
    if (!q || !k || !v || !q_norm_w || !k_norm_w || !sinks || !k_cache || !v_cache || !cache_len || !out)
        return fail(FLINT_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(out, 16))
        return fail(FLINT_ERR_INVALID_ARG, "q, k, v, the caches and out must be 16-byte aligned");
    if (!aligned(q_norm_w, 4) || !aligned(k_norm_w, 4) || !aligned(sinks, 4) || !aligned(cache_len, 4) ||
        (lse && !aligned(lse, 4)))
        return fail(FLINT_ERR_INVALID_ARG, "misaligned 32-bit array");
    const size_t need = flint::decode_workspace_bytes(B, cap, window);
    if (!workspace || !aligned(workspace, 256))
        return fail(FLINT_ERR_WORKSPACE, "workspace missing or not 256-byte aligned");
    if (workspace_bytes < need)
        return fail(FLINT_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
    int sms = 0;
    flint_status_t st = device_setup(&sms);
    if (st != FLINT_OK) return st;
    return flint::run_decode(q, k, v, q_norm_w, k_norm_w, sinks, k_cache, v_cache, cache_len, B, cap,
                             window, use_rope, rope_theta, eps, out, lse, workspace, workspace_bytes,
                             stream);
}

size_t flint_attn_bwd_workspace_bytes(int32_t T) {
    if (T < 0 || T > FLINT_MAX_TOKENS) return 0;
    return flint::bwd_workspace_bytes(T);
}

flint_status_t flint_attn_bwd(const void* q, const void* k, const void* v, const float* q_norm_w,
                              const float* k_norm_w, const float* sinks, const int32_t* pos_ids,
                              const int32_t* cu_seqlens, int32_t num_docs, const uint8_t* pad_mask,
                              int32_t batch, int32_t seqlen, int32_t T, int32_t window,
                              int32_t use_rope, float rope_theta, float eps, const void* out,
                              const float* lse, const void* dout, float* dq, float* dk, float* dv,
                              float* dq_norm_w, float* dk_norm_w, float* dsinks, void* workspace,
                              size_t workspace_bytes, void* stream) {
    NvtxRange r("flint_attn_bwd");
    g_err[0] = '\0';
    if (T < 0 || T > FLINT_MAX_TOKENS)
        return fail(FLINT_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, FLINT_MAX_TOKENS);
    if (window < 0) return fail(FLINT_ERR_INVALID_ARG, "window=%d < 0", window);
    if (use_rope != 0 && use_rope != 1) return fail(FLINT_ERR_INVALID_ARG, "use_rope must be 0 or 1");
    if (!(eps > 0.f) || !std::isfinite(eps)) return fail(FLINT_ERR_INVALID_ARG, "eps must be > 0");
    if (use_rope && (!(rope_theta > 1.f) || !std::isfinite(rope_theta)))
        return fail(FLINT_ERR_INVALID_ARG, "rope_theta must be > 1");
    if (cu_seqlens && pad_mask)
        return fail(FLINT_ERR_INVALID_ARG, "give at most one of cu_seqlens and pad_mask");
    if (cu_seqlens && (num_docs < 0 || num_docs > FLINT_MAX_TOKENS))
        return fail(FLINT_ERR_INVALID_ARG, "num_docs=%d", num_docs);
    if (pad_mask && (batch < 1 || seqlen < 1 || (long long)batch * seqlen != (long long)T))
        return fail(FLINT_ERR_INVALID_ARG, "pad_mask needs batch*seqlen == T (%d*%d vs %d)", batch,
                    seqlen, T);
    if (!dq_norm_w || !dk_norm_w || !dsinks) return fail(FLINT_ERR_INVALID_ARG, "null gradient pointer");
    if (!aligned(dq_norm_w, 4) || !aligned(dk_norm_w, 4) || !aligned(dsinks, 4))
        return fail(FLINT_ERR_INVALID_ARG, "misaligned 32-bit array");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        cudaError_t e = cudaMemsetAsync(dq_norm_w, 0, sizeof(float) * kHD, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dk_norm_w, 0, sizeof(float) * kHD, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dsinks, 0, sizeof(float) * kHQ, s);
        if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
        return FLINT_OK;
    }
    if (!q || !k || !v || !q_norm_w || !k_norm_w || !sinks || !out || !lse || !dout || !dq || !dk || !dv)
        return fail(FLINT_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
        return fail(FLINT_ERR_INVALID_ARG, "q, k, v, out, dout, dq, dk and dv must be 16-byte aligned");
    if (!aligned(q_norm_w, 4) || !aligned(k_norm_w, 4) || !aligned(sinks, 4) || !aligned(lse, 4) ||
        (pos_ids && !aligned(pos_ids, 4)) || (cu_seqlens && !aligned(cu_seqlens, 4)))
        return fail(FLINT_ERR_INVALID_ARG, "misaligned 32-bit array");
    const size_t need = flint::bwd_workspace_bytes(T);
    if (!workspace || !aligned(workspace, 256))
        return fail(FLINT_ERR_WORKSPACE, "workspace missing or not 256-byte aligned");
    if (workspace_bytes < need)
        return fail(FLINT_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
    int sms = 0;
    flint_status_t st = device_setup(&sms);
    if (st != FLINT_OK) return st;
    return flint::run_bwd(q, k, v, q_norm_w, k_norm_w, sinks, pos_ids, cu_seqlens, num_docs, pad_mask,
                          batch, seqlen, T, window, use_rope, rope_theta, eps, out, lse, dout, dq, dk, dv,
                          dq_norm_w, dk_norm_w, dsinks, workspace, sms, stream);
}

flint_status_t flint_attn_device_status(const void* workspace, void* stream) {
    if (!workspace) return fail(FLINT_ERR_WORKSPACE, "workspace is null");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
    int st = 0;
    e = cudaMemcpy(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(FLINT_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    return static_cast<flint_status_t>(st);
}

}  // extern "C"
