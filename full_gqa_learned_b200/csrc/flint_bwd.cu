// Gradient of the sink-aware GQA attention forward (sm_100a).
//
// The pages make every head's sink a trainable FP32 parameter ("flint" model
// page on NeMo AutoModel, "Parallelism and backends": the sink adjoint, and
// FA4 rejecting learned sinks in backward).  The gradient is the exact
// derivative of the forward (FlintAttention.forward on the "flint.layers" API
// page; the sink as a zero-value softmax column, HF discussion #26 on
// RecursiveSI/flint) for a loss on `out`:
//
//   D_i   = dO_i . out_i
//   P_ij  = exp(s_ij - lse_i),  s_ij = q~_i . k~_j / sqrt(128)
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dq~_i = sum_j dS_ij k~_j / sqrt(128)      dk~_j = sum_{h,i} dS_ij q~_i / sqrt(128)
//   dv_j  = sum_{h,i} P_ij dO_i               dsink_h = -sum_i exp(sink_h - lse_i) D_i
//
// then back through RoPE (rotation by -p) and RMSNorm (weight form):
//   dw += dn * x r,   dx = r w dn - x r^3 (sum_c w_c dn_c x_c) / 128.
//
// Kernels, in stream order:
//   bwd_segments_kernel  document bounds of every token (THD boundaries or a
//                        trailing-padding mask), validated
//   bwd_prep_kernel      q~, k~ as the tensor cores' FP16 operands (scaled by
//                        2^eq, 2^ek as in the forward) and D per (token, head)
//   bwd_dq_tc_kernel,    the three products on the tensor cores
//   bwd_dkv_tc_kernel    (flint_bwd_tc.cu): dq~, dk~ and dv
//   bwd_adjoint_kernel   a warp per row: the RoPE and RMSNorm adjoints of dq~
//                        and dk~, zero rows for padding, and per-CTA partial
//                        sums of dq_norm_w, dk_norm_w and dsinks
//   bwd_finish_kernel    sums the per-CTA partials in a fixed order
//                        (deterministic)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "../../include/flint_attn.h"
#include "flint_common.cuh"

namespace flint {

constexpr int kBwdThreads = 256;            // 8 warps: the query heads of one KV head
constexpr int kBwdMaxBlocks = 2048;         // grid cap; sizes the partial-sum arrays
constexpr int kBwdPartQ = kHD + kHQ;        // per-CTA partial: dq_norm_w[128], dsinks[32]
constexpr int kBwdSegThreads = 1024;

struct BwdLayout {
    size_t seg_lo, seg_hi, flags, delta, qh, kh, part_q, part_k, total;
};

// Header: status word (offset 0), the tensor-core kernels' unit counters
// (offsets 16, 20); all 256 bytes are zeroed by every call.
inline BwdLayout bwd_layout(int T) {
    BwdLayout L;
    size_t o = 256;
    L.seg_lo = o; o = ws_align(o + sizeof(int) * (size_t)T, 256);
    L.seg_hi = o; o = ws_align(o + sizeof(int) * (size_t)T, 256);
    L.flags = o;  o = ws_align(o + sizeof(int) * (size_t)((T + 127) / 128) * kHKV, 256);
    L.delta = o;  o = ws_align(o + sizeof(float) * (size_t)T * kHQ, 256);
    L.qh = o;     o = ws_align(o + 2 * (size_t)T * kHQ * kHD, 1024);
    L.kh = o;     o = ws_align(o + 2 * (size_t)T * kHKV * kHD, 256);
    L.part_q = o; o = ws_align(o + sizeof(float) * (size_t)kBwdMaxBlocks * kBwdPartQ, 256);
    L.part_k = o; o = ws_align(o + sizeof(float) * (size_t)kBwdMaxBlocks * kHD, 256);
    L.total = o;
    return L;
}

struct BwdParams {
    const __nv_bfloat16* q;      // [T,32,128]
    const __nv_bfloat16* k;      // [T,4,128]
    const __nv_bfloat16* v;      // [T,4,128]
    const float* q_norm_w;
    const float* k_norm_w;
    const float* sinks;
    const int* pos_ids;
    const int* cu_seqlens;
    const uint8_t* pad_mask;
    const __nv_bfloat16* out;    // [T,4096]
    const float* lse;            // [32,T]
    const __nv_bfloat16* dout;   // [T,4096]
    float* dq;                   // [T,32,128]
    float* dk;                   // [T,4,128]
    float* dv;                   // [T,4,128]
    float* dq_norm_w;            // [128]
    float* dk_norm_w;            // [128]
    float* dsinks;               // [32]
    int* status;
    int* seg_lo;                 // [T]: first token of the token's document, -1 = padding
    int* seg_hi;                 // [T]: one past its last token
    float* delta;                // [T,32]: D
    __half* qh;                  // [T,32,128]: q~ 2^eq, FP16
    __half* kh;                  // [T,4,128]: k~ 2^ek, FP16
    float* part_q;               // [dq grid,160]
    float* part_k;               // [dk/dv grid,128]
    int T, nseg, batch, seqlen, window, use_rope, mode;
    float rope_theta, eps;
};

__device__ __forceinline__ float bf(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ void set_status(int* status, int code) { atomicCAS(status, 0, code); }

// ---- document bounds: one CTA per document (THD) or batch row (mask)
__global__ void __launch_bounds__(kBwdSegThreads) bwd_segments_kernel(const BwdParams p) {
    const int d = blockIdx.x;
    int a = 0, b = 0;
    if (p.mode == kMaskThd) {
        a = p.cu_seqlens[d];
        b = p.cu_seqlens[d + 1];
        if ((d == 0 && a != 0) || a < 0 || b < a || b > p.T) {
            if (threadIdx.x == 0) set_status(p.status, kStatusInvalid);
            return;
        }
    } else if (p.mode == kMaskPad) {
        const size_t row = (size_t)d * p.seqlen;
        int len = 0;
        for (int c = 0; c < p.seqlen; c += kBwdSegThreads) {
            const int pi = c + threadIdx.x;
            len += __syncthreads_count(pi < p.seqlen && p.pad_mask[row + pi] != 0);
        }
        int bad = 0;
        for (int c = 0; c < p.seqlen; c += kBwdSegThreads) {
            const int pi = c + threadIdx.x;
            bad |= __syncthreads_or(pi < p.seqlen && ((p.pad_mask[row + pi] != 0) != (pi < len)));
        }
        if (bad) {
            if (threadIdx.x == 0) set_status(p.status, kStatusUnsupported);
            return;
        }
        a = d * p.seqlen;
        b = a + len;
    } else {
        a = 0;
        b = p.T;
    }
    for (int t = a + threadIdx.x; t < b; t += kBwdSegThreads) {
        p.seg_lo[t] = a;
        p.seg_hi[t] = b;
    }
}

__device__ __forceinline__ int token_pos(const BwdParams& p, int t) {
    if (p.pos_ids) return p.pos_ids[t];
    const int lo = p.seg_lo[t];
    return lo >= 0 ? t - lo : 0;
}

// Normalise and rotate one row held by a warp: lane l owns channels
// l, l+32, l+64, l+96 (RoPE pairs (l, l+64) and (l+32, l+96)).
__device__ __forceinline__ void norm_rope(const float x[4], const float* w, float eps, bool rope, int pos,
                                          const double* inv, int lane, float y[4]) {
    const float ss = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const float r = rsqrtf(ss * (1.f / kHD) + eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) y[i] = x[i] * r * w[lane + 32 * i];
    if (rope) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float c, s;
            rope_cos_sin(pos, inv[lane + 32 * i], &c, &s);
            const float a = y[i], b = y[i + 2];
            y[i] = a * c - b * s;
            y[i + 2] = b * c + a * s;
        }
    }
}

__device__ __forceinline__ void load_inv_freq(double* s_inv, float theta) {
    if (threadIdx.x < 64) s_inv[threadIdx.x] = exp2(-(double)threadIdx.x / 64.0 * log2((double)theta));
}

// ---- q~, k~ (FP16 tensor-core operands) and D: one warp per row, rows =
// T*32 query rows then T*4 key rows
__global__ void __launch_bounds__(kBwdThreads) bwd_prep_kernel(const BwdParams p) {
    __shared__ double s_inv[64];
    __shared__ float s_w[2][kHD];
    __shared__ float s_scale[2];
    load_inv_freq(s_inv, p.rope_theta);
    if (threadIdx.x < kHD) {
        s_w[0][threadIdx.x] = p.q_norm_w[threadIdx.x];
        s_w[1][threadIdx.x] = p.k_norm_w[threadIdx.x];
    }
    if (threadIdx.x < 64) {
        // the forward's power-of-two pre-scales of the FP16 operands
        const float m = warp_max_abs128(threadIdx.x < 32 ? p.q_norm_w : p.k_norm_w);
        if ((threadIdx.x & 31) == 0) s_scale[threadIdx.x >> 5] = ldexpf(1.f, prescale_exponent(m));
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const size_t nq = (size_t)p.T * kHQ, nrows = nq + (size_t)p.T * kHKV;
    const size_t wstride = (size_t)gridDim.x * (kBwdThreads / 32);
    for (size_t r = (size_t)blockIdx.x * (kBwdThreads / 32) + (threadIdx.x >> 5); r < nrows; r += wstride) {
        const bool is_q = r < nq;
        const size_t row = is_q ? r : r - nq;          // q row t*32+h, or k row t*4+g
        const int t = (int)(is_q ? row / kHQ : row / kHKV);
        const __nv_bfloat16* src = is_q ? p.q : p.k;
        float x[4], y[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = bf(src, row * kHD + lane + 32 * i);
        norm_rope(x, s_w[is_q ? 0 : 1], p.eps, p.use_rope != 0, token_pos(p, t), s_inv, lane, y);
        __half* dst = (is_q ? p.qh : p.kh) + row * kHD;
        const float sc = s_scale[is_q ? 0 : 1];
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[lane + 32 * i] = __float2half_rn(y[i] * sc);
        if (is_q) {
            float d = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) d += bf(p.dout, row * kHD + lane + 32 * i) * bf(p.out, row * kHD + lane + 32 * i);
            d = warp_sum(d);
            if (lane == 0) p.delta[row] = d;
        }
    }
}

// exp(sink - lse) for one row: 0 for sink = -inf and for sink = +inf (whose
// rows have out = 0 whatever the sink, so no gradient reaches it)
__device__ __forceinline__ float sink_share(float sink, float lse) {
    if (isinf(sink)) return 0.f;
    return expf(sink - lse);
}

// Adjoint of RoPE then RMSNorm (weight form) for one row held by a warp
// (lane l owns channels l, l+32, l+64, l+96): dy, the gradient of the
// normalised, rotated row -> dx; adds dn * x * r to dw.
__device__ __forceinline__ void norm_rope_bwd(const float x[4], const float* w, float eps, bool rope, int pos,
                                              const double* inv, int lane, const float dy[4], float dx[4],
                                              float dw[4]) {
    float dn[4] = {dy[0], dy[1], dy[2], dy[3]};
    if (rope) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float c, s;
            rope_cos_sin(pos, inv[lane + 32 * i], &c, &s);
            const float a = dy[i], b = dy[i + 2];
            dn[i] = a * c + b * s;
            dn[i + 2] = b * c - a * s;
        }
    }
    float ss = 0.f, t = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        ss = fmaf(x[i], x[i], ss);
        t = fmaf(w[lane + 32 * i] * dn[i], x[i], t);
    }
    ss = warp_sum(ss);
    t = warp_sum(t);
    const float r = rsqrtf(ss * (1.f / kHD) + eps);
    const float c3 = r * r * r * t * (1.f / kHD);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        dx[i] = r * w[lane + 32 * i] * dn[i] - x[i] * c3;
        dw[i] = fmaf(dn[i] * x[i], r, dw[i]);
    }
}

// ---- the adjoints: a warp per row, T*32 query rows then T*4 key rows.
// dq and dk hold dq~ and dk~ (tensor-core kernels) and receive dq and dk;
// padded tokens get zero rows in dq, dk and dv.
__global__ void __launch_bounds__(kBwdThreads) bwd_adjoint_kernel(const BwdParams p) {
    constexpr int kWarps = kBwdThreads / 32;
    __shared__ double s_inv[64];
    __shared__ float s_w[2][kHD];
    __shared__ float s_dw[2][kWarps][kHD];
    __shared__ float s_dsink[kWarps][kHQ];      // per warp: only that warp adds to its row
    load_inv_freq(s_inv, p.rope_theta);
    if (threadIdx.x < kHD) {
        s_w[0][threadIdx.x] = p.q_norm_w[threadIdx.x];
        s_w[1][threadIdx.x] = p.k_norm_w[threadIdx.x];
    }
    for (int t = threadIdx.x; t < kWarps * kHQ; t += kBwdThreads) (&s_dsink[0][0])[t] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float dwq[4] = {0.f, 0.f, 0.f, 0.f}, dwk[4] = {0.f, 0.f, 0.f, 0.f};
    const size_t nq = (size_t)p.T * kHQ, nrows = nq + (size_t)p.T * kHKV;
    const size_t wstride = (size_t)gridDim.x * kWarps;
    for (size_t r = (size_t)blockIdx.x * kWarps + warp; r < nrows; r += wstride) {
        const bool is_q = r < nq;
        const size_t row = is_q ? r : r - nq;          // q row t*32+h, or k row t*4+g
        const int t = (int)(is_q ? row / kHQ : row / kHKV);
        float* d = (is_q ? p.dq : p.dk) + row * kHD;
        if (p.seg_lo[t] < 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                d[lane + 32 * i] = 0.f;
                if (!is_q) p.dv[row * kHD + lane + 32 * i] = 0.f;
            }
            continue;
        }
        float x[4], dy[4], dx[4];
        const __nv_bfloat16* src = is_q ? p.q : p.k;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[i] = bf(src, row * kHD + lane + 32 * i);
            dy[i] = d[lane + 32 * i];
        }
        norm_rope_bwd(x, s_w[is_q ? 0 : 1], p.eps, p.use_rope != 0, token_pos(p, t), s_inv, lane, dy, dx,
                      is_q ? dwq : dwk);
#pragma unroll
        for (int i = 0; i < 4; ++i) d[lane + 32 * i] = dx[i];
        if (is_q && lane == 0) {
            const int h = (int)(row % kHQ);
            const float sink = p.sinks[h];
            const float L = p.lse[(size_t)h * p.T + t];
            s_dsink[warp][h] += -sink_share(sink, L) * p.delta[row];
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        s_dw[0][warp][lane + 32 * i] = dwq[i];
        s_dw[1][warp][lane + 32 * i] = dwk[i];
    }
    __syncthreads();
    if (threadIdx.x < kHD) {
        float sq = 0.f, sk = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            sq += s_dw[0][w][threadIdx.x];
            sk += s_dw[1][w][threadIdx.x];
        }
        p.part_q[(size_t)blockIdx.x * kBwdPartQ + threadIdx.x] = sq;
        p.part_k[(size_t)blockIdx.x * kHD + threadIdx.x] = sk;
    } else if (threadIdx.x < kHD + kHQ) {
        float s = 0.f;
        for (int w = 0; w < kWarps; ++w) s += s_dsink[w][threadIdx.x - kHD];
        p.part_q[(size_t)blockIdx.x * kBwdPartQ + threadIdx.x] = s;
    }
}

// ---- fixed-order sums of the per-CTA partials
// One warp per output (dq_norm_w[128], dk_norm_w[128], dsinks[32]): lane l
// sums the partials b = l, l + 32, ... in order, then the lanes' sums meet in
// a fixed shuffle tree, so every call adds in the same order.
constexpr int kBwdFinishOutputs = kHD + kHD + kHQ;
__global__ void bwd_finish_kernel(const BwdParams p, int grid_q, int grid_k) {
    const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= kBwdFinishOutputs) return;
    const float* src;
    int n, stride;
    float* dst;
    if (w < kHD) {
        src = p.part_q + w; n = grid_q; stride = kBwdPartQ; dst = p.dq_norm_w + w;
    } else if (w < 2 * kHD) {
        src = p.part_k + (w - kHD); n = grid_k; stride = kHD; dst = p.dk_norm_w + (w - kHD);
    } else {
        src = p.part_q + kHD + (w - 2 * kHD); n = grid_q; stride = kBwdPartQ; dst = p.dsinks + (w - 2 * kHD);
    }
    float s = 0.f;
    for (int b = lane; b < n; b += 32) s += src[(size_t)b * stride];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) *dst = s;
}

flint_status_t set_error(flint_status_t s, const char* msg);
flint_status_t launch_bwd_tc(const void* qh, const void* kh, const void* v, const void* dout,
                             const float* q_norm_w, const float* k_norm_w, const float* lse,
                             const float* delta, const int* seg_lo, const int* seg_hi, float* dq, float* dk,
                             float* dv, int* status, int* counters, int* flags, int T, int window, int sms,
                             cudaStream_t s);

size_t bwd_workspace_bytes(int T) { return bwd_layout(T).total; }

flint_status_t run_bwd(const void* q, const void* k, const void* v, const float* q_norm_w,
                       const float* k_norm_w, const float* sinks, const int32_t* pos_ids,
                       const int32_t* cu_seqlens, int32_t num_docs, const uint8_t* pad_mask,
                       int32_t batch, int32_t seqlen, int32_t T, int32_t window, int32_t use_rope,
                       float rope_theta, float eps, const void* out, const float* lse, const void* dout,
                       float* dq, float* dk, float* dv, float* dq_norm_w, float* dk_norm_w,
                       float* dsinks, void* workspace, int sms, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    const BwdLayout L = bwd_layout(T);
    BwdParams bp;
    bp.q = static_cast<const __nv_bfloat16*>(q);
    bp.k = static_cast<const __nv_bfloat16*>(k);
    bp.v = static_cast<const __nv_bfloat16*>(v);
    bp.q_norm_w = q_norm_w;
    bp.k_norm_w = k_norm_w;
    bp.sinks = sinks;
    bp.pos_ids = use_rope ? pos_ids : nullptr;
    bp.cu_seqlens = cu_seqlens;
    bp.pad_mask = pad_mask;
    bp.out = static_cast<const __nv_bfloat16*>(out);
    bp.lse = lse;
    bp.dout = static_cast<const __nv_bfloat16*>(dout);
    bp.dq = dq;
    bp.dk = dk;
    bp.dv = dv;
    bp.dq_norm_w = dq_norm_w;
    bp.dk_norm_w = dk_norm_w;
    bp.dsinks = dsinks;
    bp.status = reinterpret_cast<int*>(ws);
    bp.seg_lo = reinterpret_cast<int*>(ws + L.seg_lo);
    bp.seg_hi = reinterpret_cast<int*>(ws + L.seg_hi);
    bp.delta = reinterpret_cast<float*>(ws + L.delta);
    bp.qh = reinterpret_cast<__half*>(ws + L.qh);
    bp.kh = reinterpret_cast<__half*>(ws + L.kh);
    bp.part_q = reinterpret_cast<float*>(ws + L.part_q);
    bp.part_k = reinterpret_cast<float*>(ws + L.part_k);
    bp.T = T;
    bp.batch = batch;
    bp.seqlen = seqlen;
    bp.window = window;
    bp.use_rope = use_rope;
    bp.rope_theta = rope_theta;
    bp.eps = eps;
    int nseg = 1;
    bp.mode = kMaskSingle;
    if (cu_seqlens) {
        bp.mode = kMaskThd;
        nseg = num_docs;
    } else if (pad_mask) {
        bp.mode = kMaskPad;
        nseg = batch;
    }
    bp.nseg = nseg;
    // the adjoint kernel: one wave of resident CTAs, capped by the partial arrays
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, bwd_adjoint_kernel, kBwdThreads, 0);
    long long ga = (long long)sms * (occ > 0 ? occ : 1);
    if (ga > kBwdMaxBlocks) ga = kBwdMaxBlocks;
    const long long rows_all = (long long)T * (kHQ + kHKV);
    if (ga > (rows_all + 7) / 8) ga = (rows_all + 7) / 8;
    const int grid_a = (int)ga;

    cudaError_t e = cudaMemsetAsync(ws, 0, 256, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(bp.seg_lo, 0xff, sizeof(int) * (size_t)T, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws + L.flags, 0, sizeof(int) * (size_t)((T + 127) / 128) * kHKV, s);
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: workspace reset failed");
    if (nseg > 0) {
        bwd_segments_kernel<<<nseg, kBwdSegThreads, 0, s>>>(bp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: segment launch failed");
    }
    const size_t rows = (size_t)T * (kHQ + kHKV);
    size_t prep_grid = (rows + kBwdThreads / 32 - 1) / (kBwdThreads / 32);
    if (prep_grid > (size_t)sms * 16) prep_grid = (size_t)sms * 16;
    bwd_prep_kernel<<<(unsigned)prep_grid, kBwdThreads, 0, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: prep launch failed");
    flint_status_t st = launch_bwd_tc(bp.qh, bp.kh, v, dout, q_norm_w, k_norm_w, lse, bp.delta, bp.seg_lo,
                                      bp.seg_hi, dq, dk, dv, bp.status, reinterpret_cast<int*>(ws + 16),
                                      reinterpret_cast<int*>(ws + L.flags), T, window, sms, s);
    if (st != FLINT_OK) return st;
    bwd_adjoint_kernel<<<grid_a, kBwdThreads, 0, s>>>(bp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: adjoint launch failed");
    bwd_finish_kernel<<<(kBwdFinishOutputs + 7) / 8, 256, 0, s>>>(bp, grid_a, grid_a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(FLINT_ERR_CUDA, "backward: finish launch failed");
    return FLINT_OK;
}

}  // namespace flint
