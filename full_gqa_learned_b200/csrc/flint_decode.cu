// One decode step of the sink-aware GQA attention against a key/value cache
// (sm_100a, CUDA cores: the step reads each cached key and value once and is
// bound by memory, not by the tensor cores).
//
// Sequence b's new token sits at position p = cache_len[b].  Its queries and
// key get the prologue of FlintAttention.forward (NeMo AutoModel
// "flint.layers" API page): per-head RMSNorm in weight form, then NeoX RoPE at
// p on sliding layers.  It attends to the keys of positions lo .. p (lo =
// max(0, p - W + 1) on a sliding layer, the window counting the current
// token; 0 on a full layer) and to the learned sink, a zero-value softmax
// column in natural-logit units (HF discussion #26 on RecursiveSI/flint).
// Position j lives in cache slot j mod cap, so a cache of capacity >= W is a
// ring on sliding layers (the "flint" model page: a hybrid KV cache must
// honour per-layer window sizes).  The step appends the new token: its
// normalised, rotated key (rounded to BF16) and its value go to slot p mod cap.
//
// This file: the CUDA-core path (any norm weights) and the host side;
// flint_decode_tc.cu holds the tensor-core path taken when the logit bound
// is <= 48.  Both write partials in the same format and fold them with
// decode_fold (flint_decode.cuh).
//
// Split-KV: item (s, g, b) takes keys lo + 256 s .. lo + 256 s + 255 of KV
// head g and writes a partial (m, l, O) per query head in log2 units; the
// last split of (b, g) to finish folds the partials and the sink:
//   M = max(sink * log2e, max_s m_s)
//   L = 2^(sink * log2e - M) + sum_s l_s 2^(m_s - M)
//   out = sum_s O_s 2^(m_s - M) / L,  lse = (M ln 2 + ln L)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "../../include/flint_attn.h"
#include "flint_common.cuh"
#include "flint_decode.cuh"
#include "sm100.cuh"

namespace flint {

constexpr int kDecKeys = 256;          // keys per split
constexpr int kDecThreads = 128;       // split kernel: 2 keys per thread for the scores

// 6 CTAs per SM (80 registers): more loads in flight than one CTA's worth
__global__ void __launch_bounds__(kDecThreads, 6)
decode_split_kernel(const DecodeParams p) {
    __shared__ __align__(16) float s_q[kHD][kGroup];   // q~ x log2(e)/sqrt(128), channel-major
    __shared__ float s_knew[kHD];              // the new token's k~ (FP32)
    __shared__ __align__(16) float s_p[kDecKeys][kGroup];   // scores, then probabilities, key-major
    __shared__ __align__(16) float s_o[kDecThreads / 2][2 * kGroup];   // second key half's PV sums
    __shared__ float s_w[2][kHD];              // q_norm_w, k_norm_w
    __shared__ double s_inv[64];
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // under a logit bound <= 48 the tensor-core tile kernel does the step
    {
        const float bnd = decode_logit_bound(p.q_norm_w, p.k_norm_w);
        if (bnd <= kDecodeBoundMax) return;
    }
    // launched as a programmatic dependent of the tile kernel (which waited
    // for the header reset before it returned): everything below comes after
    griddep_wait();
    // CTA (loop over items (s, g, b)): keys lo + 256 s .. of KV head g of
    // sequence b; the last split of (b, g) to finish folds all of them
    auto run_item = [&](const int s, const int g, const int b) {
    const int pos = p.cache_len[b];
    const int lo = p.window > 0 ? max(0, pos - p.window + 1) : 0;
    const int n = pos - lo + 1;
    float* part = p.part + (((size_t)b * kHKV + g) * p.nsplit + s) * kPartFloats;
    if (pos < 0 || pos >= FLINT_MAX_TOKENS || n > p.cap) {
        if (tid == 0) atomicCAS(p.status, 0, 1 /* FLINT_ERR_INVALID_ARG */);
        if (tid < kGroup) { part[tid] = -INFINITY; part[kGroup + tid] = 0.f; }
        return;
    }
    const int k0 = lo + kDecKeys * s, k1 = min(lo + kDecKeys * (s + 1), pos + 1);
    if (k0 >= k1) {                            // nothing in this split
        if (tid < kGroup) { part[tid] = -INFINITY; part[kGroup + tid] = 0.f; }
        return;
    }
    const bool has_new = (k1 == pos + 1);      // this split holds the new token

    s_w[0][tid] = p.q_norm_w[tid];
    s_w[1][tid] = p.k_norm_w[tid];
    if (tid < 64) s_inv[tid] = exp2(-(double)tid / 64.0 * log2((double)p.rope_theta));
    __syncthreads();

    // ---- q~ for the 8 heads of group g (warp w: heads 2w, 2w+1); k~ of the new token
    const float qscale = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int h = 2 * warp + hh;
        float y[4];
        dec_norm_rope_row(p.q + ((size_t)b * kHQ + kGroup * g + h) * kHD, s_w[0], p.eps, p.use_rope != 0,
                          pos, s_inv, lane, y);
#pragma unroll
        for (int i = 0; i < 4; ++i) s_q[lane + 32 * i][h] = y[i] * qscale;
    }
    if (has_new && warp == 0) {
        float y[4];
        dec_norm_rope_row(p.k + ((size_t)b * kHKV + g) * kHD, s_w[1], p.eps, p.use_rope != 0, pos, s_inv,
                          lane, y);
        const size_t slot = (size_t)(pos % p.cap);
        __nv_bfloat16* kdst = p.k_cache + (((size_t)b * kHKV + g) * p.cap + slot) * kHD;
        __nv_bfloat16* vdst = p.v_cache + (((size_t)b * kHKV + g) * p.cap + slot) * kHD;
        const __nv_bfloat16* vsrc = p.v + ((size_t)b * kHKV + g) * kHD;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s_knew[lane + 32 * i] = y[i];
            kdst[lane + 32 * i] = __float2bfloat16_rn(y[i]);
            vdst[lane + 32 * i] = vsrc[lane + 32 * i];
        }
    }
    __syncthreads();

    // ---- scores: thread t takes keys k0 + t and k0 + t + 128, all 8 heads
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        const int j = tid + kDecThreads * half, kj = k0 + j;
        float acc[kGroup];
#pragma unroll
        for (int h = 0; h < kGroup; ++h) acc[h] = (kj < k1) ? 0.f : -INFINITY;
        if (kj < k1 && kj == pos) {
#pragma unroll 4
            for (int c = 0; c < kHD; ++c) {
                const float kc = s_knew[c];
                const float4 qa = *reinterpret_cast<const float4*>(&s_q[c][0]);
                const float4 qb = *reinterpret_cast<const float4*>(&s_q[c][4]);
                acc[0] = fmaf(qa.x, kc, acc[0]); acc[1] = fmaf(qa.y, kc, acc[1]);
                acc[2] = fmaf(qa.z, kc, acc[2]); acc[3] = fmaf(qa.w, kc, acc[3]);
                acc[4] = fmaf(qb.x, kc, acc[4]); acc[5] = fmaf(qb.y, kc, acc[5]);
                acc[6] = fmaf(qb.z, kc, acc[6]); acc[7] = fmaf(qb.w, kc, acc[7]);
            }
        } else if (kj < k1) {
            const uint4* krow = reinterpret_cast<const uint4*>(
                p.k_cache + (((size_t)b * kHKV + g) * p.cap + (size_t)(kj % p.cap)) * kHD);
            // the whole 256-byte row in flight at once
            uint4 kr[kHD / 8];
#pragma unroll
            for (int c8 = 0; c8 < kHD / 8; ++c8) kr[c8] = krow[c8];
#pragma unroll
            for (int c8 = 0; c8 < kHD / 8; ++c8) {
                const uint4 u = kr[c8];
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float kc = (e & 1) ? __uint_as_float(w4[e >> 1] & 0xffff0000u)
                                             : __uint_as_float(w4[e >> 1] << 16);
                    const int c = 8 * c8 + e;
                    const float4 qa = *reinterpret_cast<const float4*>(&s_q[c][0]);
                    const float4 qb = *reinterpret_cast<const float4*>(&s_q[c][4]);
                    acc[0] = fmaf(qa.x, kc, acc[0]); acc[1] = fmaf(qa.y, kc, acc[1]);
                    acc[2] = fmaf(qa.z, kc, acc[2]); acc[3] = fmaf(qa.w, kc, acc[3]);
                    acc[4] = fmaf(qb.x, kc, acc[4]); acc[5] = fmaf(qb.y, kc, acc[5]);
                    acc[6] = fmaf(qb.z, kc, acc[6]); acc[7] = fmaf(qb.w, kc, acc[7]);
                }
            }
        }
        *reinterpret_cast<float4*>(&s_p[j][0]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(&s_p[j][4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    __syncthreads();

    // ---- per head: max over the split, probabilities, sum (warp w: heads 2w, 2w+1)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int h = 2 * warp + hh;
        float x[kDecKeys / 32], mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < kDecKeys / 32; ++i) { x[i] = s_p[lane + 32 * i][h]; mx = fmaxf(mx, x[i]); }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < kDecKeys / 32; ++i) {
            const float e = exp2f(x[i] - mx);        // keys past the split: 2^-inf = 0
            s_p[lane + 32 * i][h] = e;
            sum += e;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) { part[h] = mx; part[kGroup + h] = sum; }
    }
    __syncthreads();

    // ---- O_h[c] = sum_j p_h[j] V_j[c]: thread t takes channels 2(t % 64),
    // +1 over half of the split's keys; the two halves meet in shared memory
    {
        const int cp = tid & 63, kh = tid >> 6;
        float o[kGroup][2];
#pragma unroll
        for (int h = 0; h < kGroup; ++h) o[h][0] = o[h][1] = 0.f;
        const int nk = k1 - k0;
        const int jb = kh * (kDecKeys / 2), je = min(nk, jb + kDecKeys / 2);
        const uint32_t* vnew = reinterpret_cast<const uint32_t*>(p.v + ((size_t)b * kHKV + g) * kHD) + cp;
        const uint32_t* vbase = reinterpret_cast<const uint32_t*>(p.v_cache + ((size_t)b * kHKV + g) * p.cap * kHD) + cp;
        const size_t slot_stride = (size_t)kHD / 2;               // 32-bit words per cache slot
        int slot = (k0 + jb) % p.cap;                             // advances by one per key
#pragma unroll 16
        for (int jj = jb; jj < je; ++jj) {
            const int kk = k0 + jj;
            const uint32_t v2 = (kk == pos) ? *vnew : vbase[(size_t)slot * slot_stride];
            slot = (slot + 1 == p.cap) ? 0 : slot + 1;
            const float v0 = __uint_as_float(v2 << 16), v1 = __uint_as_float(v2 & 0xffff0000u);
            const float4 pa = *reinterpret_cast<const float4*>(&s_p[jj][0]);
            const float4 pb = *reinterpret_cast<const float4*>(&s_p[jj][4]);
            const float pr[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                o[h][0] = fmaf(pr[h], v0, o[h][0]);
                o[h][1] = fmaf(pr[h], v1, o[h][1]);
            }
        }
        if (kh == 1) {
#pragma unroll
            for (int h = 0; h < kGroup; ++h) { s_o[cp][2 * h] = o[h][0]; s_o[cp][2 * h + 1] = o[h][1]; }
        }
        __syncthreads();
        if (kh == 0) {
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                const float2 r = make_float2(o[h][0] + s_o[cp][2 * h], o[h][1] + s_o[cp][2 * h + 1]);
                *reinterpret_cast<float2*>(&part[2 * kGroup + h * kHD + 2 * cp]) = r;
            }
        }
    }
    };
    const int n_items = p.nsplit * kHKV * p.B;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int s = item % p.nsplit, g = (item / p.nsplit) % kHKV, b = item / (p.nsplit * kHKV);
        run_item(s, g, b);
        // this split's partial is written: the last of the (b, g) splits folds
        __threadfence();
        __syncthreads();
        if (tid == 0) s_last = atomicAdd(p.arrive + b * kHKV + g, 1) == p.nsplit - 1;
        __syncthreads();
        if (s_last) {
            __threadfence();
            decode_fold(p, b, g, p.nsplit, tid);
        }
        __syncthreads();
    }
}

flint_status_t set_error(flint_status_t s, const char* msg);

// Zeroes the status word, the tile kernel's work counter and the
// split-arrival counters of one call.  The tile kernel is launched as its
// programmatic dependent: its setup overlaps this, and it waits for this
// grid before it touches those words.
__global__ void decode_zero_kernel(int* hdr, int n_words) {
    griddep_launch_dependents();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_words; i += gridDim.x * blockDim.x) hdr[i] = 0;
}

size_t decode_nsplit(int cap, int window) {
    const int nmax = window > 0 ? (window < cap ? window : cap) : cap;
    return (size_t)((nmax + kDecKeys - 1) / kDecKeys);
}

size_t decode_workspace_bytes(int B, int cap, int window) {
    const size_t ns = decode_nsplit(cap, window), nt = (size_t)decode_tc_nsplit(cap);
    return decode_header_bytes(B) + (size_t)B * kHKV * (ns > nt ? ns : nt) * kPartFloats * sizeof(float);
}

flint_status_t launch_decode_tc(const DecodeParams& p, int sms, cudaStream_t s);

flint_status_t run_decode(const void* q, const void* k, const void* v, const float* q_norm_w,
                          const float* k_norm_w, const float* sinks, void* k_cache, void* v_cache,
                          const int32_t* cache_len, int32_t B, int32_t cap, int32_t window,
                          int32_t use_rope, float rope_theta, float eps, void* out, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream) {
    DecodeParams dp;
    dp.q = static_cast<const __nv_bfloat16*>(q);
    dp.k = static_cast<const __nv_bfloat16*>(k);
    dp.v = static_cast<const __nv_bfloat16*>(v);
    dp.q_norm_w = q_norm_w;
    dp.k_norm_w = k_norm_w;
    dp.sinks = sinks;
    dp.k_cache = static_cast<__nv_bfloat16*>(k_cache);
    dp.v_cache = static_cast<__nv_bfloat16*>(v_cache);
    dp.cache_len = cache_len;
    dp.out = static_cast<__nv_bfloat16*>(out);
    dp.lse = lse;
    dp.status = static_cast<int*>(workspace);
    dp.arrive = reinterpret_cast<int*>(static_cast<char*>(workspace) + 256);
    dp.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + decode_header_bytes(B));
    dp.B = B;
    dp.cap = cap;
    dp.window = window;
    dp.use_rope = use_rope;
    dp.nsplit = (int)decode_nsplit(cap, window);
    dp.nsplit_tc = decode_tc_nsplit(cap);
    dp.rope_theta = rope_theta;
    dp.eps = eps;
    (void)workspace_bytes;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // status word, the tile kernel's work counter, the split-arrival counters
    const int hdr_words = (int)(decode_header_bytes(B) / sizeof(int));
    const int zgrid = (hdr_words + 255) / 256 < 64 ? (hdr_words + 255) / 256 : 64;
    decode_zero_kernel<<<zgrid, 256, 0, s>>>(dp.status, hdr_words);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "decode: status reset failed");
    // Both kernels are enqueued, each a programmatic dependent of the launch
    // before it, so their launches and setup overlap the work ahead of them;
    // each decides from the norm weights whether it runs (the tile kernel
    // under a logit bound <= 48) and the other returns at once.  Each writes
    // the output itself (the last split of a sequence and KV head folds them
    // all).
    int sms = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    flint_status_t st = launch_decode_tc(dp, sms > 0 ? sms : 1, s);
    if (st != FLINT_OK) return st;
    // two CTAs per SM loop over the items (when the tile kernel runs, these
    // only read the weights and return)
    const long long items = (long long)dp.nsplit * kHKV * B;
    const long long cap_grid = 2LL * (sms > 0 ? sms : 1);
    const int grid = (int)(items < cap_grid ? items : cap_grid);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_split_kernel, dp);
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "decode: split launch failed");
    return FLINT_OK;
}

}  // namespace flint
