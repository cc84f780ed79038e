// Definitions shared by the decode kernels (flint_decode.cu: the CUDA-core
// split kernel and the combine kernel; flint_decode_tc.cu: the tensor-core
// tile kernel).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "flint_common.cuh"

namespace flint {

__device__ __forceinline__ float dec_bf16(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Normalise (weight form) and, if rope, rotate one 128-channel row held by a
// warp: lane l owns channels l, l+32, l+64, l+96 (the pairs (l, l+64) and
// (l+32, l+96) rotate with frequencies l and l+32).  Returns the 4 values.
// The same on values already loaded (x[i] = channel lane + 32 i).
__device__ __forceinline__ void dec_norm_rope_vals(const float x[4], const float* w, float eps, bool rope, int pos,
                                                   const double* inv_freq, int lane, float y[4]) {
    float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rn = rsqrtf(ss * (1.f / kHD) + eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) y[i] = x[i] * rn * w[lane + 32 * i];
    if (rope) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float c, s;
            rope_cos_sin(pos, inv_freq[lane + 32 * i], &c, &s);
            const float a = y[i], b = y[i + 2];
            y[i] = a * c - b * s;
            y[i + 2] = b * c + a * s;
        }
    }
}
__device__ __forceinline__ void dec_load_row(const __nv_bfloat16* row, int lane, float x[4]) {
    const uint16_t* r16 = reinterpret_cast<const uint16_t*>(row);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = dec_bf16(r16[lane + 32 * i]);
}
__device__ __forceinline__ void dec_norm_rope_row(const __nv_bfloat16* row, const float* w, float eps,
                                                  bool rope, int pos, const double* inv_freq, int lane,
                                                  float y[4]) {
    float x[4];
    dec_load_row(row, lane, x);
    dec_norm_rope_vals(x, w, eps, rope, pos, inv_freq, lane, y);
}

struct DecodeParams {
    const __nv_bfloat16* q;      // [B,32,128]
    const __nv_bfloat16* k;      // [B,4,128]
    const __nv_bfloat16* v;      // [B,4,128]
    const float* q_norm_w;
    const float* k_norm_w;
    const float* sinks;
    __nv_bfloat16* k_cache;      // [B,4,cap,128] (head-major)
    __nv_bfloat16* v_cache;      // [B,4,cap,128]
    const int* cache_len;        // [B]
    __nv_bfloat16* out;          // [B,4096]
    float* lse;                  // [32,B]
    int* status;                 // device status word
    int* arrive;                 // [B, 4] splits of (b, g) done (zeroed per call)
    float* part;                 // [B,4,nsplit,8,(2 + 128)]: per split m[8], l[8]
                                 // (log2 units) and O[8][128] unnormalised
    int B, cap, window, use_rope;
    int nsplit;                  // splits of the CUDA-core kernel (by position)
    int nsplit_tc;               // splits of the tensor-core kernel (by cache slot)
    float rope_theta, eps;
};

constexpr int kPartFloats = 8 * (2 + kHD);   // m[8], l[8], O[8][128]


// Bound on every scaled logit of a decode step (log2 units): |q~|_2 <=
// sqrt(128) max|w_q| and |k~|_2 <= sqrt(128) max|w_k| (1 + 2^-9) for a key
// rounded to BF16 in the cache, so |q~ . k~| / sqrt(128) log2(e) <= 16.3222
// (1 + 2^-9) max|w_q| max|w_k|; 16.45 leaves a margin.  The tensor-core tile
// kernel starts every softmax at this bound and needs it <= 48 (every term
// 2^(s - bound) then stays a normal FP32 and BF16); otherwise the CUDA-core
// split kernel runs.  Every decode kernel decides the same way from the
// weights.
__device__ __forceinline__ float decode_logit_bound(const float* q_norm_w, const float* k_norm_w) {
    const float mq = warp_max_abs128(q_norm_w);
    const float mk = warp_max_abs128(k_norm_w);
    return 16.45f * mq * mk + 1e-3f;
}
constexpr float kDecodeBoundMax = 48.f;

// Workspace: status word (offset 0), the tile kernel's item counter (4),
// per (sequence, KV head) split-arrival counters (256 ..), then the partials.
// The first decode_header_bytes(B) bytes are zeroed by every call.
__host__ __device__ inline size_t decode_header_bytes(int B) {
    return 256 + ((size_t)B * kHKV * sizeof(int) + 255) / 256 * 256;
}

// Folds the splits of (b, g) with the sinks of its 8 query heads into the
// output and the LSE (thread c of 128: channel c):
//   M = max(sink log2e, max_s m_s),  L = 2^(sink log2e - M) + sum_s l_s 2^(m_s - M),
//   out = sum_s O_s 2^(m_s - M) / L,  lse = M ln 2 + ln L.
// The partials were written by other CTAs: read through L2.
__device__ __forceinline__ void decode_fold(const DecodeParams& p, int b, int g, int nsplit, int c) {
    const float* base = p.part + ((size_t)b * kHKV + g) * nsplit * kPartFloats;
    for (int hh = 0; hh < kGroup; ++hh) {
        const int h = kGroup * g + hh;
        const float sink = p.sinks[h];
        float acc = 0.f, L = 0.f, M;
        if (sink == INFINITY) {
            M = INFINITY;
        } else {
            M = sink * 1.4426950408889634f;
            for (int s = 0; s < nsplit; ++s) M = fmaxf(M, __ldcg(base + s * kPartFloats + hh));
            if (M > -INFINITY) {
                L = (sink > -INFINITY) ? exp2f(sink * 1.4426950408889634f - M) : 0.f;
                for (int s = 0; s < nsplit; ++s) {
                    const float* ps = base + s * kPartFloats;
                    const float ms = __ldcg(ps + hh);
                    if (ms == -INFINITY) continue;
                    const float a = exp2f(ms - M);
                    L += __ldcg(ps + kGroup + hh) * a;
                    acc += __ldcg(ps + 2 * kGroup + hh * kHD + c) * a;
                }
            }
        }
        const float o = (L > 0.f) ? acc / L : 0.f;
        p.out[((size_t)b * kHQ + h) * kHD + c] = __float2bfloat16_rn(o);
        if (c == 0 && p.lse) {
            float v;
            if (M == INFINITY) v = INFINITY;
            else if (L > 0.f) v = M * 0.6931471805599453f + logf(L);
            else v = -INFINITY;
            p.lse[(size_t)h * p.B + b] = v;
        }
    }
}

// Tensor-core decode: the cache is read in tiles of 128 slots; a split is a
// run of consecutive tiles of one (sequence, KV head).
constexpr int kDtSlots = 128;
__host__ __device__ inline int decode_tc_tiles(int cap) { return (cap + kDtSlots - 1) / kDtSlots; }
__host__ __device__ inline int decode_tc_nsplit(int cap) {
    const int nt = decode_tc_tiles(cap);
    const int per = nt > 128 ? (nt + 15) / 16 : 8;    // at most 16 splits, at least 8 tiles each
    return (nt + per - 1) / per;
}
__host__ __device__ inline int decode_tc_tiles_per_split(int cap) {
    const int nt = decode_tc_tiles(cap), ns = decode_tc_nsplit(cap);
    return (nt + ns - 1) / ns;
}

}  // namespace flint
