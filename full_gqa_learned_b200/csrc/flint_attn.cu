// Sink-aware causal GQA attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Computes, for every valid query token i and query head h (KV head g = h/8),
//   out[i,h,:] = sum_j e^{s_ij} v[j,g,:] / (e^{sink_h} + sum_j e^{s_ij}),
//   lse[h,i]   = ln(e^{sink_h} + sum_j e^{s_ij}),
// with s_ij = q~_i . k~_j / sqrt(128) over the keys j of the same document,
// j <= i, and i - j < window on sliding layers.  q~ is q after the weight-form
// RMSNorm and, on sliding layers, NeoX RoPE (FlintAttention.forward and
// _apply_rope on the NeMo AutoModel "flint.layers" API page; the sink as an
// extra zero-value softmax column in natural-logit units: HF discussion #26 on
// RecursiveSI/flint).  q~ and k~ (FP16, scaled by powers of two) were
// prepared by the preparation kernel; q~ sits in the output rows of its own
// token, which each tile reads through TMA before it writes its result there.
//
// Layout of one CTA (one per SM, persistent, 384 threads):
//   warp 0      dynamic scheduler + TMA producer (Q tiles, K/V chunks)
//   warp 1      TMEM owner; lane 0 issues every tcgen05.mma and commit
//   warps 2-3   idle (their registers go to the softmax warpgroups)
//   warps 4-7   softmax warpgroup of tile 0 (tokens q0..q0+15)
//   warps 8-11  softmax warpgroup of tile 1 (tokens q0+16..q0+31)
// A tile is 128 MMA rows = 16 tokens x the 8 query heads of one KV group, so
// every K/V chunk in shared memory serves 8 heads x 32 tokens.
//
// Tensor memory (512 columns): S_t at column 128 t, O_t at 256 + 128 t.  P_t
// (BF16) overwrites the first 64 columns of S_t and feeds the PV MMA straight
// from TMEM.  The online softmax starts from m = sink*log2(e), l = 1, which
// is exactly the extra sink column; the running max is only raised (and O
// rescaled) when it grows by more than 2^8, so the rescale is rare.
// Interior chunks after the first skip the row max altogether while the row
// sum of their terms stays within 2^8; masked chunks treat each 32-column
// block as full, empty or partial.  Each softmax warp stores its 4 output
// tokens through a swizzled staging block and TMA.  The kernel runs as a
// programmatic dependent of the preparation kernel: its setup overlaps that
// kernel's tail and it reads nothing prepared before griddepcontrol.wait.
#include <cuda.h>
#include <cmath>
#include "flint_common.cuh"
#include "sm100.cuh"

namespace flint {

constexpr int kThreads = 384;
constexpr uint32_t kRegsControl = 80;
constexpr uint32_t kRegsSoftmax = 208;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= 384 * 168, "register split");
constexpr uint32_t kTileBytes = 128 * kHD * 2;       // 32 KiB: 128 rows x 128 x 16-bit
constexpr uint32_t kHalfTile = kTileBytes / 2;       // one 64-column swizzled half

// Shared memory plan (offsets from a 1024-aligned base).
constexpr uint32_t kOffQ = 0;                        // 2 Q tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;   // 2 K stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;   // 2 V stages
constexpr uint32_t kOffStage = kOffV + 2 * kTileBytes;       // output staging, 4 KiB per softmax warp
constexpr uint32_t kStageBytes = 32 * 128;                   // 32 rows x 64 channels x BF16
constexpr uint32_t kOffBar = kOffStage + 8 * kStageBytes;    // mbarriers
constexpr uint32_t kNumBars = 32;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kOffInvFreq = kOffMisc + 64;              // 64 RoPE inverse frequencies (double)
constexpr uint32_t kOffWq = kOffInvFreq + 64 * 8;            // q_norm weight (128 floats)
constexpr uint32_t kSmemUsed = kOffWq + kHD * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;            // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per block");
// RoPE table of one softmax warp's 4 tokens in its staging block: per token,
// 32 frequency pairs (f, f+1) as {cos f, cos f+1, sin f, sin f+1} (16 bytes
// each), then the 32 pairs {-sin f, -sin f+1} (8 bytes each); rows padded
// by 16 bytes against bank conflicts (784 = 49 x 16 keeps every row 16-byte
// aligned)
constexpr uint32_t kTabCs = 32 * 16;
constexpr uint32_t kTabStride = kTabCs + 32 * 8 + 16;
static_assert(kTabStride % 16 == 0, "16-byte aligned table rows");
static_assert(4 * kTabStride <= kStageBytes, "RoPE table fits the staging block");

// barrier indices
enum : uint32_t {
    B_SCHED_FULL = 0, B_SCHED_EMPTY = 2,
    B_Q_FULL = 4, B_Q_EMPTY = 8,
    B_K_FULL = 10, B_K_EMPTY = 12, B_V_FULL = 14, B_V_EMPTY = 16,
    B_S_FULL = 18, B_P_FULL = 20, B_O_FULL = 22, B_DRAIN = 24,
    B_TEST_WAIT = 26,    // nothing arrives here: the timeout test hook waits on it
    B_Q_READY = 28       // the tile's queries normalised in place (128 arrivals)
};

struct Misc {
    int sched[2];
    uint32_t tmem_base;
    int abort_flag;
    float logit_scale;   // log2(e)/sqrt(128) * 2^-(eq+ek)
    float q_scale;       // 2^eq
    float logit_bound;   // bound on every scaled logit (log2 units), or +inf
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Coefficients of the degree-4 polynomial for 2^f on [-1/2, 1/2], written by
// exp2_poly_fit.py (max relative error 2.6e-6).
constexpr float kExp2C0 = 9.999992847e-01f;
constexpr float kExp2C1 = 6.931217909e-01f;
constexpr float kExp2C2 = 2.402474433e-01f;
constexpr float kExp2C3 = 5.591785908e-02f;
constexpr float kExp2C4 = 9.570101276e-03f;

// Packed FP32 pairs (Blackwell f32x2 arithmetic): one instruction acts on both
// halves of a 64-bit register.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float f2_lo(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo;
}
__device__ __forceinline__ float f2_hi(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return hi;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x for a pair of finite x <= 64 on the FMA and integer pipes (results below
// 2^-126 flush towards 2^-126).  Cody-Waite split x = n + f with n rounded to
// nearest by the 1.5*2^23 shifter (the float t = x + shifter holds n in its
// low mantissa bits), degree-4 polynomial for 2^f on [-1/2, 1/2], then n
// added to the exponent field.  Because 0x4B400000 << 23 vanishes modulo 2^32,
// adding (bits(t) << 23) adds n << 23.  Takes load off the MUFU unit.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
    x = f2(fmaxf(f2_lo(x), -126.f), fmaxf(f2_hi(x), -126.f));
    const uint64_t sh = f2(12582912.f, 12582912.f);          // 1.5 * 2^23
    const uint64_t nsh = f2(-12582912.f, -12582912.f);
    const uint64_t neg1 = f2(-1.f, -1.f);
    const uint64_t t = f2_add(x, sh);
    const uint64_t n = f2_add(t, nsh);
    const uint64_t f = f2_fma(n, neg1, x);                   // in [-1/2, 1/2]
    uint64_t q = f2_fma(f2(kExp2C4, kExp2C4), f, f2(kExp2C3, kExp2C3));
    q = f2_fma(q, f, f2(kExp2C2, kExp2C2));
    q = f2_fma(q, f, f2(kExp2C1, kExp2C1));
    q = f2_fma(q, f, f2(kExp2C0, kExp2C0));
    const float p0 = __int_as_float(__float_as_int(f2_lo(q)) + (__float_as_int(f2_lo(t)) << 23));
    const float p1 = __int_as_float(__float_as_int(f2_hi(q)) + (__float_as_int(f2_hi(t)) << 23));
    return f2(p0, p1);
}

// Pairs j of each 16-pair block with (j % 8) < kPolyPairs take the polynomial.
// Measured costs per warp instruction and scheduler on B200: ex2 8 cycles;
// fma/add.f32x2, cvt.rn.bf16x2.f32 and 3-input max 2 each (cvt and max share
// a pipe, ex2 overlaps all of them); a polynomial pair costs ~20 on the
// FMA/ALU pipes.  Shares of 2/8 and 3/8 measured slower than 1/8.
constexpr int kPolyPairs = 1;

// Two FP32 values -> packed BF16 pair, `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ int chunk_cols(int ks, int ke) {
    int n = ke - ks;
    n = n > kKeyChunk ? kKeyChunk : n;
    return (n + 15) & ~15;
}

// Two FP32 values -> packed 16-bit pair for the PV operand and the output:
// BF16, or FP16 under the FP16 attention-compute policy.
template <bool F16>
__device__ __forceinline__ uint32_t pack_pv(float lo, float hi) {
    if constexpr (F16) {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&h);
    } else {
        return pack_bf16(lo, hi);
    }
}

// The kernel body.
// QPREP: the queries arrive normalised and rotated in FP16 from the
//   preparation kernel instead of being prepared on tile load.  Sliding
//   layers use it: their units are 5 chunks long, too short to hide the
//   prologue between a unit's last chunk and its epilogue.
// F16 (implies QPREP): the FP16 attention-compute policy ("flint" model page,
//   "Numerical comparison": normalised, rotated Q/K/V cast to FP16 for the
//   attention): values are FP16, P and the output are FP16, and the softmax
//   keeps its exact running max (P stays within FP16's normal range).
template <bool QPREP, bool F16>
__device__ __forceinline__ void attn_fwd_body(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                              const CUtensorMap& tm_v, const CUtensorMap& tm_o,
                                              const CUtensorMap& tm_o1, const AttnParams& p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kOffBar;
    auto bar = [&](uint32_t i) { return bar0 + 8u * i; };
    Misc* misc = reinterpret_cast<Misc*>(smem + kOffMisc);
    volatile int* abort_flag = &misc->abort_flag;

    const WsLayout L = ws_layout(p.T, p.nseg);
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(p.ws + L.header);
    const int4* items = reinterpret_cast<const int4*>(p.ws + L.items);
    int* status = &hdr->status;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---------------------------------------------------------------- setup
    if (tid == 0) {
        mbar_init(bar(B_SCHED_FULL + 0), 1);
        mbar_init(bar(B_SCHED_FULL + 1), 1);
        // released by the MMA thread and by lane 0 of each of the 8 softmax warps
        mbar_init(bar(B_SCHED_EMPTY + 0), 1 + 8);
        mbar_init(bar(B_SCHED_EMPTY + 1), 1 + 8);
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(B_Q_FULL + t), 1);
            mbar_init(bar(B_Q_EMPTY + t), 1);
            mbar_init(bar(B_K_FULL + t), 1);
            mbar_init(bar(B_K_EMPTY + t), 1);
            mbar_init(bar(B_V_FULL + t), 1);
            mbar_init(bar(B_V_EMPTY + t), 1);
            mbar_init(bar(B_S_FULL + t), 1);
            mbar_init(bar(B_P_FULL + t), 128);      // every softmax thread of tile t
            mbar_init(bar(B_O_FULL + t), 1);
            mbar_init(bar(B_Q_READY + t), 128);     // every softmax thread of tile t
        }
        mbar_init(bar(B_DRAIN), 1);
        mbar_init(bar(B_TEST_WAIT), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&misc->tmem_base), 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        const float mq = warp_max_abs128(p.q_norm_w);
        const float mk = warp_max_abs128(p.k_norm_w);
        if (lane == 0) {
            const int eq = prescale_exponent(mq), ek = prescale_exponent(mk);
            misc->logit_scale = ldexpf(1.4426950408889634f * 0.08838834764831845f, -(eq + ek));
            misc->q_scale = ldexpf(1.f, eq);
            // After the weight-form RMSNorm a head row has |x / rms(x)|_2 <=
            // sqrt(128), so |q~|_2 <= sqrt(128) max|w_q| and likewise for k~;
            // RoPE preserves the norm.  Every logit q~.k~ / sqrt(128) is then
            // within sqrt(128) max|w_q| max|w_k|, i.e. log2(e) sqrt(128) =
            // 16.3222 times that in log2 units (16.35: margin for the FP16
            // rounding of both operands).  When that bound is small enough
            // that 2^(s - bound) stays a normal FP32 for every logit s
            // (bound <= 48), the online softmax starts its running max at the
            // bound: no row max and no rescale on any chunk.
            const float bnd = 16.35f * mq * mk + 1e-3f;
            misc->logit_bound = (!F16 && bnd <= 48.f) ? bnd : INFINITY;
        }
    }
    if (warp == 3) {
        // q_norm weight and the RoPE inverse frequencies theta^(-f/64), f < 64
        float* wq = reinterpret_cast<float*>(smem + kOffWq);
        double* inv_freq = reinterpret_cast<double*>(smem + kOffInvFreq);
#pragma unroll
        for (int i = 0; i < 4; ++i) wq[lane + 32 * i] = p.q_norm_w[lane + 32 * i];
        const double l2t = log2((double)p.rope_theta);
        inv_freq[lane] = exp2(-(double)lane / 64.0 * l2t);
        inv_freq[lane + 32] = exp2(-(double)(lane + 32) / 64.0 * l2t);
    }
    // everything above overlaps the tail of the preparation kernel; the work
    // plan and the prepared keys and queries are read only after it completed
    griddep_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const int n_units = hdr->n_items * p.ng;

    // Registers: launched with 384 x 168 = 64512.  Warps 0-3 (producer, MMA,
    // two idle) drop to kRegsControl, the two softmax warpgroups rise to
    // kRegsSoftmax; 128*80 + 256*208 = 63488 <= 64512.
    if (warp < 4) {
      regs_dec<kRegsControl>();
      if (warp == 0) {
        // ============================================================ producer
        if (lane == 0) {
            uint32_t sslot = 0, sph = 0, qph = 0, kst = 0, kph = 0, vst = 0, vph = 0;
            uint32_t narm_q = 0, narm_k = 0, narm_v = 0;   // loads armed so far
            // Units are taken one ahead of the loads (the next unit is known
            // while the current one streams).
            int u = atomicAdd(&hdr->counter, 1);
            if (u >= n_units) u = -1;
            for (;;) {
                if (!mbar_wait(bar(B_SCHED_EMPTY + sslot), sph ^ 1, abort_flag, status)) break;
                misc->sched[sslot] = u;
                mbar_arrive(bar(B_SCHED_FULL + sslot));
                sslot ^= 1; if (sslot == 0) sph ^= 1;
                if (u < 0) break;
                int un = atomicAdd(&hdr->counter, 1);
                if (un >= n_units) un = -1;
                const int4 it = items[u / p.ng];
                const int g = u % p.ng;
                const int q0 = it.x, nq = it.y, ds = it.z, nch = it.w;
                bool ok = true;
                for (int t = 0; t < 2 && ok; ++t) {
                    ok = mbar_wait(bar(B_Q_EMPTY + t), qph ^ 1, abort_flag, status);
                    if (!ok) break;
                    const uint32_t dst = sbase + kOffQ + t * kTileBytes;
                    mbar_expect_tx(bar(B_Q_FULL + t), kTileBytes);
                    tma_load_3d(dst, &tm_q, bar(B_Q_FULL + t), 0, kGroup * g, q0 + kTokPerTile * t);
                    tma_load_3d(dst + kHalfTile, &tm_q, bar(B_Q_FULL + t), 64, kGroup * g,
                                q0 + kTokPerTile * t);
                }
                if (!ok) break;
                ++narm_q;
                qph ^= 1;
                const int ke = q0 + nq;
                const int kb = p.window > 0 ? max(ds, q0 - p.window + 1) : ds;
                (void)ke;
                for (int c = 0; c < nch && ok; ++c) {
                    const int ks = kb + kKeyChunk * c;
                    ok = mbar_wait(bar(B_K_EMPTY + kst), kph ^ 1, abort_flag, status);
                    if (!ok) break;
                    uint32_t dst = sbase + kOffK + kst * kTileBytes;
                    mbar_expect_tx(bar(B_K_FULL + kst), kTileBytes);
                    tma_load_3d(dst, &tm_k, bar(B_K_FULL + kst), 0, g, ks);
                    tma_load_3d(dst + kHalfTile, &tm_k, bar(B_K_FULL + kst), 64, g, ks);
                    ++narm_k;
                    kst ^= 1; if (kst == 0) kph ^= 1;
                    ok = mbar_wait(bar(B_V_EMPTY + vst), vph ^ 1, abort_flag, status);
                    if (!ok) break;
                    dst = sbase + kOffV + vst * kTileBytes;
                    mbar_expect_tx(bar(B_V_FULL + vst), kTileBytes);
                    tma_load_3d(dst, &tm_v, bar(B_V_FULL + vst), 0, g, ks);
                    tma_load_3d(dst + kHalfTile, &tm_v, bar(B_V_FULL + vst), 64, g, ks);
                    ++narm_v;
                    vst ^= 1; if (vst == 0) vph ^= 1;
                }
                if (!ok) break;
                u = un;
            }
            // drain: every armed load has landed before shared memory is released
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            volatile int never = 0;
            for (int t = 0; t < 2; ++t)
                if (narm_q) mbar_wait(bar(B_Q_FULL + t), (narm_q - 1) & 1, &never, nullptr, lim);
            for (uint32_t s = 0; s < 2; ++s) {
                // stage s received loads number s, s+2, s+4, ...
                const uint32_t nk = (narm_k + 1 - s) / 2, nv = (narm_v + 1 - s) / 2;
                if (nk) mbar_wait(bar(B_K_FULL + s), (nk - 1) & 1, &never, nullptr, lim);
                if (nv) mbar_wait(bar(B_V_FULL + s), (nv - 1) & 1, &never, nullptr, lim);
            }
        }
      } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_f16(F16 ? 0u : 1u, F16 ? 0u : 1u, 1, 128);
            // Descriptor words.  Only the low word (start address) changes
            // between MMAs; the issuing thread shares its scheduler with two
            // busy softmax warps, so each MMA is kept to a 32-bit add and the
            // instruction itself.
            const uint64_t dq0 = smem_desc_sw128(sbase + kOffQ, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sbase + kOffK, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + kOffV, kHalfTile, 1024);
            const uint32_t q_lo = (uint32_t)dq0, q_hi = (uint32_t)(dq0 >> 32);
            const uint32_t k_lo = (uint32_t)dk0, k_hi = (uint32_t)(dk0 >> 32);
            const uint32_t v_lo = (uint32_t)dv0, v_hi = (uint32_t)(dv0 >> 32);
            constexpr uint32_t kTileStep = kTileBytes >> 4;
            uint32_t sslot = 0, sph = 0, qrph = 0, kst = 0, kph = 0, vst = 0, vph = 0, pph = 0;
            auto issue_s = [&](uint32_t t, uint32_t kstage, int ncols) {
                const uint32_t idesc = idesc_f16(0, 0, 0, (uint32_t)ncols);
                const uint32_t qa = q_lo + t * kTileStep, kb_ = k_lo + kstage * kTileStep;
                const uint32_t d = tmem + 128u * t;
#pragma unroll
                for (uint32_t kk = 0; kk < kHD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (kHalfTile >> 4) + (kk & 3) * 2;
                    mma_ss_w(d, qa + off, q_hi, kb_ + off, k_hi, idesc, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](uint32_t t, uint32_t vstage, int ncols, bool acc) {
                const uint32_t vb = v_lo + vstage * kTileStep;
                const uint32_t d = tmem + 256u + 128u * t, pa = tmem + 128u * t;
                const int nk = ncols >> 4;
                mma_ts_w(d, pa, vb, v_hi, idesc_pv, acc ? 1u : 0u);
#pragma unroll
                for (int kk = 1; kk < 8; ++kk)
                    if (kk < nk) mma_ts_w(d, pa + 8u * kk, vb + kk * (2048 >> 4), v_hi, idesc_pv, 1u);
            };
            // test hook: a wait that runs out (FLINT_ERR_TIMEOUT and abort)
            // before any MMA is issued
            const bool stalled =
                p.test_wait_ns > 0 && !mbar_wait(bar(B_TEST_WAIT), 0, abort_flag, status, p.test_wait_ns);
            for (; !stalled;) {
                if (!mbar_wait(bar(B_SCHED_FULL + sslot), sph, abort_flag, status)) break;
                const int u = misc->sched[sslot];
                mbar_arrive(bar(B_SCHED_EMPTY + sslot));
                sslot ^= 1; if (sslot == 0) sph ^= 1;
                if (u < 0) break;
                const int4 it = items[u / p.ng];
                const int q0 = it.x, nq = it.y, ds = it.z, nch = it.w;
                const int ke = q0 + nq;
                const int kb = p.window > 0 ? max(ds, q0 - p.window + 1) : ds;
                // S for chunk 0, each tile as soon as its Q tile has landed
                if (!mbar_wait(bar(B_K_FULL + kst), kph, abort_flag, status)) break;
                if (!mbar_wait(bar(B_Q_READY + 0), qrph, abort_flag, status)) break;
                tc_fence_after();
                int ncol = chunk_cols(kb, ke);
                issue_s(0, kst, ncol);
                mma_commit(bar(B_S_FULL + 0));
                if (!mbar_wait(bar(B_Q_READY + 1), qrph, abort_flag, status)) break;
                tc_fence_after();
                qrph ^= 1;
                issue_s(1, kst, ncol);
                mma_commit(bar(B_S_FULL + 1));
                if (nch == 1) {
                    mma_commit(bar(B_Q_EMPTY + 0));
                    mma_commit(bar(B_Q_EMPTY + 1));
                }
                mma_commit(bar(B_K_EMPTY + kst));
                kst ^= 1; if (kst == 0) kph ^= 1;
                bool ok = true;
                for (int c = 0; c < nch && ok; ++c) {
                    const int nc_cur = ncol;
                    int nc_next = 0;
                    if (c + 1 < nch) nc_next = chunk_cols(kb + kKeyChunk * (c + 1), ke);
                    ok = mbar_wait(bar(B_V_FULL + vst), vph, abort_flag, status);
                    if (!ok) break;
                    ok = mbar_wait(bar(B_P_FULL + 0), pph, abort_flag, status);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(0, vst, nc_cur, c > 0);
                    if (c + 1 < nch) {
                        ok = mbar_wait(bar(B_K_FULL + kst), kph, abort_flag, status);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(0, kst, nc_next);
                        mma_commit(bar(B_S_FULL + 0));
                        if (c + 2 == nch) mma_commit(bar(B_Q_EMPTY + 0));
                    } else {
                        mma_commit(bar(B_O_FULL + 0));
                    }
                    ok = mbar_wait(bar(B_P_FULL + 1), pph, abort_flag, status);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(1, vst, nc_cur, c > 0);
                    mma_commit(bar(B_V_EMPTY + vst));
                    vst ^= 1; if (vst == 0) vph ^= 1;
                    if (c + 1 < nch) {
                        issue_s(1, kst, nc_next);
                        mma_commit(bar(B_S_FULL + 1));
                        if (c + 2 == nch) mma_commit(bar(B_Q_EMPTY + 1));
                        mma_commit(bar(B_K_EMPTY + kst));
                        kst ^= 1; if (kst == 0) kph ^= 1;
                    } else {
                        mma_commit(bar(B_O_FULL + 1));
                    }
                    pph ^= 1;
                    ncol = nc_next;
                }
                if (!ok) break;
            }
            // drain: every MMA issued so far has completed
            mma_commit(bar(B_DRAIN));
            volatile int never = 0;
            mbar_wait(bar(B_DRAIN), 0, &never, nullptr, 100ull * 1000ull * 1000ull);
        }
      }
    } else {
        regs_inc<kRegsSoftmax>();
        // ============================================================ softmax
        const int t = (warp - 4) >> 2;               // tile 0 or 1
        const int r = tid - 128 - 128 * t;           // row = TMEM lane, 0..127
        const int tl = r >> 3, hl = r & 7;           // token within tile, head within group
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u;
        const uint32_t t_s = tmem + (lane_base << 16) + 128u * t;
        const uint32_t t_o = tmem + (lane_base << 16) + 256u + 128u * t;
        const float C = misc->logit_scale;
        const float LB = misc->logit_bound;
        uint32_t sslot = 0, sph = 0, s_ph = 0, oph = 0, qph = 0;
        // this warp's output staging: its 32 rows = tokens 4*(warp&3) .. +3
        // of the tile, 64 channels at a time; it also holds the RoPE table of
        // those 4 tokens while a new query tile is prepared
        uint8_t* stg = smem + kOffStage + (warp - 4) * kStageBytes;
        const uint32_t stg_s = sbase + kOffStage + (warp - 4) * kStageBytes;
        // Warps of the warpgroup run without block-level barriers; every
        // wait's outcome is made warp-uniform (tcgen05.ld/st are
        // .sync.aligned) and a warp that gives up simply leaves the loop.
        auto fetch_unit = [&](int* u_out) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SCHED_FULL + sslot), sph, abort_flag, status)))
                return false;
            *u_out = misc->sched[sslot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SCHED_EMPTY + sslot));
            sslot ^= 1; if (sslot == 0) sph ^= 1;
            return true;
        };
        // Query prologue of unit `un` on this tile (FlintAttention.forward on
        // the "flint.layers" API page: q_norm, then _apply_rope on sliding
        // layers; model page "Model Architecture": normalisation precedes
        // RoPE).  The producer loaded the raw BF16 rows by TMA into this
        // tile's Q slot (128-byte swizzle, row r = token r/8, head r%8);
        // thread r normalises row r (weight-form RMSNorm with eps), rotates
        // channel pairs (f, f+64) by pos * theta^(-f/64) when RoPE is on,
        // scales by 2^eq and writes it back in place as FP16, the QK^T
        // operand.  This runs between the unit's last softmax chunk and its
        // epilogue, while the tensor pipe works on the last PV MMAs.
        auto prepare_q = [&](const int un) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(bar(B_Q_FULL + t), qph, abort_flag, status)))
                return false;
            qph ^= 1;
            if constexpr (QPREP) {
                // the preparation kernel already normalised and rotated them
                mbar_arrive(bar(B_Q_READY + t));
                return true;
            }
            const int4 itn = items[un / p.ng];
            const int tok = itn.x + kTokPerTile * t + tl;
            const uint8_t* tab = stg + (lane >> 3) * kTabStride;
            if (p.use_rope) {
                // this warp's 4 tokens x 32 frequency pairs, lane (token, head
                // hl) computing pairs 4 hl .. 4 hl + 3; the block is free once
                // lane 0's earlier output stores have read it
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
                int pos = 0;
                if (tok < p.T) pos = p.pos_ids ? p.pos_ids[tok] : tok - itn.z;
                const double* inv_freq = reinterpret_cast<const double*>(smem + kOffInvFreq);
                uint8_t* tw = stg + (lane >> 3) * kTabStride;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int pp = 4 * hl + e;                       // pair (2 pp, 2 pp + 1)
                    float c0, s0, c1, s1;
                    rope_cos_sin(pos, inv_freq[2 * pp], &c0, &s0);
                    rope_cos_sin(pos, inv_freq[2 * pp + 1], &c1, &s1);
                    *reinterpret_cast<float4*>(tw + 16 * pp) = make_float4(c0, c1, s0, s1);
                    *reinterpret_cast<float2*>(tw + kTabCs + 8 * pp) = make_float2(-s0, -s1);
                }
                __syncwarp();
            }
            uint8_t* qrow = smem + kOffQ + t * kTileBytes + r * 128;
            const int swz = r & 7;
            // pass 1: sum of squares of the row (16 x 16 bytes)
            uint64_t ss2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 a = *reinterpret_cast<const uint4*>(qrow + (c >> 3) * kHalfTile + (((c & 7) ^ swz) << 4));
                const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t v2 = f2(__uint_as_float(av[j] << 16), __uint_as_float(av[j] & 0xFFFF0000u));
                    ss2[j] = f2_fma(v2, v2, ss2[j]);
                }
            }
            const uint64_t sst = f2_add(f2_add(ss2[0], ss2[1]), f2_add(ss2[2], ss2[3]));
            const float rn = rsqrtf((f2_lo(sst) + f2_hi(sst)) * (1.f / kHD) + p.eps) * misc->q_scale;
            const uint64_t rn2 = f2(rn, rn);
            const float* wq = reinterpret_cast<const float*>(smem + kOffWq);
            // pass 2: channels 8c .. 8c+7 of each half per step, as pairs
            // (f, f+1) in packed FP32; y = Rot(x w) rn, written back in place
            // as FP16
#pragma unroll 2
            for (int c = 0; c < 8; ++c) {
                uint8_t* pa = qrow + ((c ^ swz) << 4);
                uint8_t* pb = pa + kHalfTile;
                const uint4 a = *reinterpret_cast<const uint4*>(pa);
                const uint4 b = *reinterpret_cast<const uint4*>(pb);
                const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
                const float4 w0a = *reinterpret_cast<const float4*>(wq + 8 * c);
                const float4 w0b = *reinterpret_cast<const float4*>(wq + 8 * c + 4);
                const float4 w1a = *reinterpret_cast<const float4*>(wq + 64 + 8 * c);
                const float4 w1b = *reinterpret_cast<const float4*>(wq + 64 + 8 * c + 4);
                const uint64_t w0[4] = {f2(w0a.x, w0a.y), f2(w0a.z, w0a.w), f2(w0b.x, w0b.y), f2(w0b.z, w0b.w)};
                const uint64_t w1[4] = {f2(w1a.x, w1a.y), f2(w1a.z, w1a.w), f2(w1b.x, w1b.y), f2(w1b.z, w1b.w)};
                uint32_t h0[4], h1[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    const uint64_t x0 = f2(__uint_as_float(av[e2] << 16), __uint_as_float(av[e2] & 0xFFFF0000u));
                    const uint64_t x1 = f2(__uint_as_float(bv[e2] << 16), __uint_as_float(bv[e2] & 0xFFFF0000u));
                    uint64_t n0 = f2_mul(x0, w0[e2]);
                    uint64_t n1 = f2_mul(x1, w1[e2]);
                    if (p.use_rope) {
                        const int pp = 4 * c + e2;
                        const float4 cs = *reinterpret_cast<const float4*>(tab + 16 * pp);
                        const float2 ns = *reinterpret_cast<const float2*>(tab + kTabCs + 8 * pp);
                        const uint64_t cc = f2(cs.x, cs.y), sn = f2(cs.z, cs.w), nsn = f2(ns.x, ns.y);
                        const uint64_t y0 = f2_fma(n1, nsn, f2_mul(n0, cc));   // n0 cos - n1 sin
                        const uint64_t y1 = f2_fma(n0, sn, f2_mul(n1, cc));    // n1 cos + n0 sin
                        n0 = y0;
                        n1 = y1;
                    }
                    n0 = f2_mul(n0, rn2);
                    n1 = f2_mul(n1, rn2);
                    const __half2 lo = __floats2half2_rn(f2_lo(n0), f2_hi(n0));
                    const __half2 hi = __floats2half2_rn(f2_lo(n1), f2_hi(n1));
                    h0[e2] = *reinterpret_cast<const uint32_t*>(&lo);
                    h1[e2] = *reinterpret_cast<const uint32_t*>(&hi);
                }
                *reinterpret_cast<uint4*>(pa) = make_uint4(h0[0], h0[1], h0[2], h0[3]);
                *reinterpret_cast<uint4*>(pb) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
            }
            // generic-proxy writes -> the tensor core's (async proxy) reads
            fence_proxy_async_smem();
            mbar_arrive(bar(B_Q_READY + t));
            return true;
        };
        int u = -1;
        bool ok = fetch_unit(&u);
        if (ok && u >= 0) ok = prepare_q(u);
        while (ok && u >= 0) {
            const int4 it = items[u / p.ng];
            const int g = u % p.ng;
            const int q0 = it.x, nq = it.y, ds = it.z, nch = it.w;
            const int h = kGroup * g + hl;
            const int tok0 = q0 + kTokPerTile * t;
            const int i = tok0 + tl;
            const bool row_valid = (kTokPerTile * t + tl) < nq;
            const int ke = q0 + nq;
            const int kb = p.window > 0 ? max(ds, q0 - p.window + 1) : ds;

            // ---- online softmax over the key chunks.  The sink is the
            // extra zero-value column: m starts at sink * log2(e) with l = 1,
            // or, with a logit bound, at max(sink, bound) with l the sink's
            // term 2^(sink - m)
            const float sink = p.sinks[h];
            const float sink_l2 = sink * 1.4426950408889634f;   // log2 domain
            const bool bnd = __all_sync(0xffffffffu, LB < INFINITY && sink_l2 < INFINITY);
            float m, l;
            if (bnd) {
                m = fmaxf(sink_l2, LB);
                l = ex2(sink_l2 - m);
            } else {
                m = sink_l2;
                l = (sink == -INFINITY) ? 0.f : 1.f;
            }
            const int lo = p.window > 0 ? i - p.window + 1 : -(1 << 30);
            bool alive = true;
            for (int c = 0; c < nch; ++c) {
                const int ks = kb + kKeyChunk * c;
                const int nc = chunk_cols(ks, ke);
                const int nblk = (nc + 31) >> 5;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + t), s_ph, abort_flag, status));
                if (!ok) { alive = false; break; }
                s_ph ^= 1;
                tc_fence_after();
                const bool boundary = (c == nch - 1) || (ks + nc - 1 > tok0) ||
                                      (p.window > 0 && ks < tok0 + kTokPerTile - p.window);
                // Interior chunks after the first with a finite running max,
                // and every interior chunk under a logit bound, take the fast
                // path below (no row max).
                const bool fastp =
                    !boundary && (bnd || (c > 0 && __all_sync(0xffffffffu, m > -INFINITY && m < INFINITY)));
                // S columns of this chunk, one TMEM load per 32 columns.  On
                // the fast path the exponentials of columns 0..63 overlap the
                // load of columns 64..127.
                uint32_t sv[128];
                tmem_ld32(t_s, sv);
                if (nblk > 1) tmem_ld32(t_s + 32u, sv + 32);
                if (fastp) tmem_wait_ld();
                if (nblk > 2) tmem_ld32(t_s + 64u, sv + 64);
                if (nblk > 3) tmem_ld32(t_s + 96u, sv + 96);
                if (!fastp) tmem_wait_ld();
                // Row r sees columns jlo .. jhi of the chunk.  Each block of 32
                // columns is, for the whole warp, either full (no mask),
                // empty (P = 0, nothing to compute) or partial (masked per
                // element); interior chunks are full.
                const int jlo = lo - ks, jhi = min(i - ks, nc - 1);
                uint32_t fullm = 0xFu, emptym = 0u;
                if (boundary) {
                    const int lo_max = __reduce_max_sync(0xffffffffu, jlo);
                    const int lo_min = __reduce_min_sync(0xffffffffu, jlo);
                    const int hi_max = __reduce_max_sync(0xffffffffu, jhi);
                    const int hi_min = __reduce_min_sync(0xffffffffu, jhi);
                    fullm = 0u;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        if (lo_max <= 32 * b && hi_min >= 32 * b + 31) fullm |= 1u << b;
                        else if (hi_max < 32 * b || lo_min > 32 * b + 31) emptym |= 1u << b;
                    }
                }
                // row max over the S columns: 3-input max, 8 independent
                // chains; masked columns become -inf in sv
                auto row_max_full = [&]() -> float {
                    float mxp[8];
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8) mxp[k8] = -INFINITY;
#pragma unroll
                    for (int j = 0; j < 128; j += 2)
                        mxp[(j >> 1) & 7] = max3(mxp[(j >> 1) & 7], __uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
                    return max3(max3(mxp[0], mxp[1], mxp[2]), max3(mxp[3], mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]));
                };
                auto row_max = [&]() -> float {
                    float mxp[8];
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8) mxp[k8] = -INFINITY;
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        if (fullm & (1u << b)) {
#pragma unroll
                            for (int j = 32 * b; j < 32 * b + 32; j += 2)
                                mxp[(j >> 1) & 7] = max3(mxp[(j >> 1) & 7], __uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
                        } else if (!(emptym & (1u << b))) {
#pragma unroll
                            for (int j = 32 * b; j < 32 * b + 32; j += 2) {
                                const float x0 = ((j >= jlo) && (j <= jhi)) ? __uint_as_float(sv[j]) : -INFINITY;
                                const float x1 = ((j + 1 >= jlo) && (j + 1 <= jhi)) ? __uint_as_float(sv[j + 1]) : -INFINITY;
                                sv[j] = __float_as_uint(x0);
                                sv[j + 1] = __float_as_uint(x1);
                                mxp[(j >> 1) & 7] = max3(mxp[(j >> 1) & 7], x0, x1);
                            }
                        }
                    }
                    return max3(max3(mxp[0], mxp[1], mxp[2]), max3(mxp[3], mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]));
                };
                // masked columns become -inf in sv (no row max)
                auto apply_mask = [&]() {
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        if (!(fullm & (1u << b)) && !(emptym & (1u << b))) {
#pragma unroll
                            for (int j = 32 * b; j < 32 * b + 32; ++j)
                                if (j < jlo || j > jhi) sv[j] = __float_as_uint(-INFINITY);
                        }
                    }
                };
                // Raise the running max to cover mx (always on the first
                // chunk, where m still holds the sink; later only when it grew
                // by more than 2^8) and rescale l and O.  Returns whether any
                // row of the warp raised.
                auto raise_to = [&](float mx) -> bool {
                    const float m_new = fmaxf(m, mx * C);
                    const bool raise = (c == 0) ? (m_new > m) : (m_new > m + 8.f);
                    float alpha = 1.f;
                    if (raise) {
                        alpha = ex2(m - m_new);
                        l *= alpha;
                    }
                    const bool any = __any_sync(0xffffffffu, raise);
                    // rescale O in TMEM (warp-uniform: tcgen05.ld/st are .sync.aligned)
                    if (c > 0 && any) {
#pragma unroll 1
                        for (int b = 0; b < 8; ++b) {
                            uint32_t v[16];
                            tmem_ld16(t_o + 16u * b, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
                            tmem_st16(t_o + 16u * b, v);
                        }
                    }
                    if (raise) m = m_new;
                    return any;
                };
                // P = 2^(s*C - m) -> BF16 into the first 64 columns of S;
                // returns the row sum.  Interior chunks: all 128 columns, and
                // with `poly` (finite m) part of the pairs go through the
                // polynomial.
                auto exp_full = [&](bool poly) -> float {
                    const float negm = (m == -INFINITY) ? 0.f : -m;
                    const uint64_t C2 = f2(C, C), negm2 = f2(negm, negm);
                    uint64_t lp[4];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) lp[k4] = 0ull;   // (+0.0f, +0.0f)
                    if (poly) {
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const uint64_t x = f2_fma(f2(__uint_as_float(sv[32 * b + 2 * j]),
                                                             __uint_as_float(sv[32 * b + 2 * j + 1])), C2, negm2);
                                uint64_t pp;
                                if ((j & 7) < kPolyPairs) pp = exp2_poly2(x);
                                else pp = f2(ex2(f2_lo(x)), ex2(f2_hi(x)));
                                lp[j & 3] = f2_add(lp[j & 3], pp);
                                pk[j] = pack_pv<F16>(f2_lo(pp), f2_hi(pp));
                            }
                            tmem_st16(t_s + 16u * b, pk);
                        }
                    } else {
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const uint64_t x = f2_fma(f2(__uint_as_float(sv[32 * b + 2 * j]),
                                                             __uint_as_float(sv[32 * b + 2 * j + 1])), C2, negm2);
                                const uint64_t pp = f2(ex2(f2_lo(x)), ex2(f2_hi(x)));
                                lp[j & 3] = f2_add(lp[j & 3], pp);
                                pk[j] = pack_pv<F16>(f2_lo(pp), f2_hi(pp));
                            }
                            tmem_st16(t_s + 16u * b, pk);
                        }
                    }
                    const uint64_t ls = f2_add(f2_add(lp[0], lp[1]), f2_add(lp[2], lp[3]));
                    return f2_lo(ls) + f2_hi(ls);
                };
                // Blocks b0 .. b1-1 with the polynomial share (unmasked, finite m).
                auto exp_part = [&](const int b0, const int b1) -> float {
                    const uint64_t C2 = f2(C, C), negm2 = f2(-m, -m);
                    uint64_t lp[4];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) lp[k4] = 0ull;   // (+0.0f, +0.0f)
#pragma unroll
                    for (int b = b0; b < b1; ++b) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint64_t x = f2_fma(f2(__uint_as_float(sv[32 * b + 2 * j]),
                                                         __uint_as_float(sv[32 * b + 2 * j + 1])), C2, negm2);
                            uint64_t pp;
                            if ((j & 7) < kPolyPairs) pp = exp2_poly2(x);
                            else pp = f2(ex2(f2_lo(x)), ex2(f2_hi(x)));
                            lp[j & 3] = f2_add(lp[j & 3], pp);
                            pk[j] = pack_pv<F16>(f2_lo(pp), f2_hi(pp));
                        }
                        tmem_st16(t_s + 16u * b, pk);
                    }
                    const uint64_t ls = f2_add(f2_add(lp[0], lp[1]), f2_add(lp[2], lp[3]));
                    return f2_lo(ls) + f2_hi(ls);
                };
                // Masked chunks: full blocks as above, partial blocks with ex2
                // (the masked -inf maps to exactly 0), empty blocks store zeros.
                auto exp_blocks = [&]() -> float {
                    const float negm = (m == -INFINITY) ? 0.f : -m;
                    const uint64_t C2 = f2(C, C), negm2 = f2(negm, negm);
                    uint64_t lp[4];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) lp[k4] = 0ull;   // (+0.0f, +0.0f)
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        uint32_t pk[16];
                        if (emptym & (1u << b)) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) pk[j] = 0u;
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const uint64_t x = f2_fma(f2(__uint_as_float(sv[32 * b + 2 * j]),
                                                             __uint_as_float(sv[32 * b + 2 * j + 1])), C2, negm2);
                                const uint64_t pp = f2(ex2(f2_lo(x)), ex2(f2_hi(x)));
                                lp[j & 3] = f2_add(lp[j & 3], pp);
                                pk[j] = pack_pv<F16>(f2_lo(pp), f2_hi(pp));
                            }
                        }
                        if (b < nblk) tmem_st16(t_s + 16u * b, pk);
                    }
                    const uint64_t ls = f2_add(f2_add(lp[0], lp[1]), f2_add(lp[2], lp[3]));
                    return f2_lo(ls) + f2_hi(ls);
                };
                float lsum = 0.f;
                if (fastp && bnd) {
                    // m is at least the logit bound: every term is at most 1
                    lsum = exp_part(0, 2);
                    tmem_wait_ld();                        // columns 64..127
                    lsum += exp_part(2, 4);
                } else if (bnd) {
                    apply_mask();
                    lsum = exp_blocks();
                } else if (fastp) {
                    // Exponentials against the current m without a row max.
                    // Every term is at most the row sum, so a sum within 2^8
                    // keeps each term inside the lazy-rescale bound.  A larger
                    // sum (rare) takes the exact max and, if some row's max
                    // moved by more than 2^8, rescales and recomputes.
#pragma unroll 1
                    for (int attempt = 0; attempt < 2; ++attempt) {
                        lsum = exp_part(0, 2);
                        tmem_wait_ld();                    // columns 64..127 (no-op when recomputing)
                        lsum += exp_part(2, 4);
                        if (attempt == 1 || !__any_sync(0xffffffffu, !(lsum <= 256.f))) break;
                        if (!raise_to(row_max_full())) break;   // first attempt stands
                        tmem_wait_st();                    // its P stores land before the new ones
                    }
                } else if (!boundary) {
                    // first chunk (m still holds the sink) or infinite max
                    raise_to(row_max_full());
                    lsum = exp_full(__all_sync(0xffffffffu, m > -INFINITY && m < INFINITY));
                } else {
                    raise_to(row_max());
                    lsum = exp_blocks();
                }
                l += lsum;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P_FULL + t));
            }
            if (!alive) break;

            // ---- the next unit: its query tile is prepared now, while the
            // tensor pipe runs this unit's last PV MMAs
            int un = -1;
            if (!fetch_unit(&un)) break;
            if (un >= 0 && !prepare_q(un)) break;

            // ---- epilogue: O / l -> BF16, LSE
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL + t), oph, abort_flag, status));
            if (!ok) break;
            oph ^= 1;
            tc_fence_after();
            const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
            // Valid tokens of this warp's 4: where a document ends inside the
            // tile, rows of other documents must not be written.
            const int wt0 = kTokPerTile * t + 4 * (warp & 3);       // first token of the warp, in the item
            const int nvw = max(0, min(4, nq - wt0));
            const int sw = lane & 7;
            // One 64-channel half at a time: O / l -> BF16 into the warp's
            // staging block in the 128-byte-swizzled layout of the output
            // tensor map, then lane 0 stores it with TMA (one 4-token box, or
            // one box per valid token).  The TMEM load of the second half
            // overlaps the store of the first.
            uint32_t pk[32];
            {
                uint32_t v[64];
                tmem_ld32(t_o, v);
                tmem_ld32(t_o + 32u, v + 32);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    pk[j] = pack_pv<F16>(__uint_as_float(v[2 * j]) * inv_l, __uint_as_float(v[2 * j + 1]) * inv_l);
            }
#pragma unroll 1
            for (int hb = 0; hb < 2; ++hb) {
                // the staging block is free once lane 0's earlier stores have read it
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ sw) << 4)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && nvw > 0) {
                    if (nvw == 4) {
                        tma_store_3d(&tm_o, stg_s, 64 * hb, kGroup * g, q0 + wt0);
                    } else {
                        for (int k = 0; k < nvw; ++k)
                            tma_store_3d(&tm_o1, stg_s + 1024u * k, 64 * hb, kGroup * g, q0 + wt0 + k);
                    }
                    bulk_commit_group();
                }
                if (hb == 0) {
                    uint32_t v[64];
                    tmem_ld32(t_o + 64u, v);
                    tmem_ld32(t_o + 96u, v + 32);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        pk[j] = pack_pv<F16>(__uint_as_float(v[2 * j]) * inv_l,
                                          __uint_as_float(v[2 * j + 1]) * inv_l);
                }
            }
            if (row_valid && p.lse) p.lse[(size_t)h * p.T + i] = m * 0.6931471805599453f + logf(l);
            tc_fence_before();
            u = un;
        }
    }

    // ---------------------------------------------------------------- teardown
    if (warp >= 4 && lane == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const __grid_constant__ CUtensorMap tm_o1, const AttnParams p) {
    attn_fwd_body<false, false>(tm_q, tm_k, tm_v, tm_o, tm_o1, p);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_qprep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ CUtensorMap tm_o1, const AttnParams p) {
    attn_fwd_body<true, false>(tm_q, tm_k, tm_v, tm_o, tm_o1, p);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_f16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ CUtensorMap tm_o1, const AttnParams p) {
    attn_fwd_body<true, true>(tm_q, tm_k, tm_v, tm_o, tm_o1, p);
}

extern const unsigned kAttnSmemBytes = kSmemBytes;
extern const unsigned kAttnThreads = kThreads;

}  // namespace flint
