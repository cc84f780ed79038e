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
// RecursiveSI/flint).  k~ was prepared by the preparation kernel.
//
// Layout of one CTA (one per SM, persistent, 384 threads):
//   warp 0      dynamic scheduler, TMA producer of K chunks
//   warp 1      TMEM owner; lane 0 issues every tcgen05.mma and commit
//   warp 2      TMA producer of V chunks
//   warp 3      TMA producer of raw Q tiles
//   warps 4-7   softmax warpgroup A: columns 0-63 of every S chunk
//   warps 8-11  softmax warpgroup B: columns 64-127 (same rows; the two
//               exchange row maxima once per chunk)
//   warps 12-15 tile warpgroup: Q prologue of the next item, epilogue of the
//               previous one
// A work item is one tile of 128 MMA rows = 16 tokens x the 8 query heads of
// one KV group, so every K/V chunk in shared memory serves 8 heads.
//
// Tensor memory (512 columns): two S buffers (columns 0 and 128), O (256),
// two buffers of the normalised FP16 Q (384 and 448).  With S double-buffered
// the MMA warp runs QK^T two chunks ahead of PV, so the softmax of chunk c
// overlaps the QK^T of chunk c+1 and the tensor pipe always has queued work.
// Q comes from TMEM (A operand), K and V from shared memory.  P (BF16)
// overwrites the first 64 columns of its S buffer and feeds the PV MMA from
// TMEM.  The online softmax starts from m = sink*log2(e), l = 1, which is
// exactly the extra sink column; the running max is only raised (and O
// rescaled) when it grows by more than 2^8, so the rescale is rare.
#include <cuda.h>
#include <cmath>
#include "flint_common.cuh"
#include "sm100.cuh"

namespace flint {

constexpr int kThreads = 512;
// Registers: launched with 512 x 128 = 65536; the control warpgroup drops to
// 64, the two softmax warpgroups rise to 160, the tile warpgroup stays at
// 128: 128 * (64 + 2 * 160 + 128) = 65536.
constexpr uint32_t kRegsControl = 64;
constexpr uint32_t kRegsSoftmax = 160;
constexpr uint32_t kRegsTile = 128;
static_assert(128 * (kRegsControl + 2 * kRegsSoftmax + kRegsTile) <= 512 * 128, "register split");

constexpr uint32_t kTileBytes = 128 * kHD * 2;       // 32 KiB: 128 rows x 128 x 16-bit
constexpr uint32_t kHalfTile = kTileBytes / 2;       // one 64-column swizzled half
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kSchedSlots = 4;

// Shared memory plan (offsets from a 1024-aligned base).
constexpr uint32_t kOffQraw = 0;                                   // raw BF16 Q tile
constexpr uint32_t kOffK = kOffQraw + kTileBytes;                  // K stages (FP16)
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;          // V stages (BF16)
constexpr uint32_t kOffRope = kOffV + kVStages * kTileBytes;       // [16][64] float2
constexpr uint32_t kRopeBytes = kTokPerTile * 64 * 8;
constexpr uint32_t kOffStats = kOffRope + kRopeBytes;              // [2][128] float4 (m, lA, lB)
constexpr uint32_t kOffPmax = kOffStats + 2 * 128 * 16;            // [2][2][128] f32 partial maxima
constexpr uint32_t kOffW = kOffPmax + 2 * 2 * 128 * 4;             // q_norm_w [128] f32
constexpr uint32_t kOffInv = kOffW + kHD * 4;                      // inv_freq [64] f64
constexpr uint32_t kOffBar = kOffInv + 64 * 8;                     // mbarriers
constexpr uint32_t kNumBars = 40;
constexpr uint32_t kOffFifo = kOffBar + kNumBars * 8;              // MMA item queue [4] int4
constexpr uint32_t kOffMisc = kOffFifo + 4 * 16;
constexpr uint32_t kSmemUsed = kOffMisc + 64;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;                  // + alignment slack

// Tensor memory columns.
constexpr uint32_t kTmemS = 0;      // S buffers at 0 and 128 (P overwrites their first 64)
constexpr uint32_t kTmemO = 256;    // O accumulator
constexpr uint32_t kTmemQ = 384;    // normalised FP16 Q buffers at 384 and 448

// barrier indices
enum : uint32_t {
    B_SCHED_FULL = 0,      // [4]
    B_SCHED_EMPTY = 4,     // [4]
    B_QRAW_FULL = 8,
    B_QRAW_EMPTY = 9,
    B_Q_READY = 10,        // [2]
    B_Q_FREE = 12,         // [2]
    B_K_FULL = 14,         // [3]
    B_K_EMPTY = 17,        // [3]
    B_V_FULL = 20,         // [2]
    B_V_EMPTY = 22,        // [2]
    B_S_FULL = 24,         // [2]
    B_P_FULL = 26,         // [2]
    B_PV_DONE = 28,        // [2]
    B_O_FULL = 30,
    B_O_FREE = 31,
    B_STATS_FULL = 32,     // [2]
    B_STATS_EMPTY = 34,    // [2]
    B_DRAIN = 36
};

struct Misc {
    int sched[kSchedSlots];
    uint32_t tmem_base;
    int abort_flag;
    float q_scale;       // 2^eq
    float logit_scale;   // log2(e)/sqrt(128) * 2^-(eq+ek)
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
// Measured costs per warp instruction and scheduler on B200: ex2 8 cycles,
// fma/add.f32x2 2, cvt.rn.bf16x2.f32 ~4.5; the polynomial pair costs ~20 on
// the FMA/ALU pipes, so MUFU and the FMA/ALU pipes balance near 1/8.
constexpr int kPolyPairs = 1;

// Two FP32 values -> packed 16-bit pair, `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// AND of a per-thread flag over the `count` threads of named barrier `id`;
// also orders their shared-memory accesses.
__device__ __forceinline__ bool block_and(uint32_t id, uint32_t count, bool ok) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)ok), "r"(id), "r"(count)
        : "memory");
    return res != 0;
}

__device__ __forceinline__ int chunk_cols(int ks, int ke) {
    int n = ke - ks;
    n = n > kKeyChunk ? kKeyChunk : n;
    return (n + 15) & ~15;
}


// One work item as seen by every role.
struct ItemView {
    int q0, nq, ds, nch, g, kb, ke;
};

__device__ __forceinline__ ItemView load_item(const int4* items, int u, int window) {
    const int4 it = items[u >> 2];
    ItemView v;
    v.q0 = it.x; v.nq = it.y; v.ds = it.z; v.nch = it.w; v.g = u & 3;
    v.ke = it.x + it.y;
    v.kb = window > 0 ? max(it.z, it.x - window + 1) : it.z;
    return v;
}

// Scheduler ring: the producer writes one work unit per slot; every consumer
// role reads the slots in order.
struct SchedCursor {
    uint32_t slot = 0, phase = 0;
    __device__ __forceinline__ void advance() {
        slot = (slot + 1) & (kSchedSlots - 1);
        if (slot == 0) phase ^= 1;
    }
};

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + kOffBar;
    auto bar = [&](uint32_t i) { return bar0 + 8u * i; };
    Misc* misc = reinterpret_cast<Misc*>(smem + kOffMisc);
    float* s_wq = reinterpret_cast<float*>(smem + kOffW);
    double* s_inv = reinterpret_cast<double*>(smem + kOffInv);
    float4* s_stats = reinterpret_cast<float4*>(smem + kOffStats);
    float* s_pmax = reinterpret_cast<float*>(smem + kOffPmax);
    int4* s_fifo = reinterpret_cast<int4*>(smem + kOffFifo);
    volatile int* abort_flag = &misc->abort_flag;

    const WsLayout L = ws_layout(p.T, p.nseg);
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(p.ws + L.header);
    const int4* items = reinterpret_cast<const int4*>(p.ws + L.items);
    int* status = &hdr->status;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---------------------------------------------------------------- setup
    if (tid == 0) {
        for (int s = 0; s < kSchedSlots; ++s) {
            mbar_init(bar(B_SCHED_FULL + s), 1);
            // MMA thread, Q and V producers, lane 0 of the 8 softmax and 4 tile warps
            mbar_init(bar(B_SCHED_EMPTY + s), 1 + 2 + 8 + 4);
        }
        mbar_init(bar(B_QRAW_FULL), 1);
        mbar_init(bar(B_QRAW_EMPTY), 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_Q_READY + b), 128);
            mbar_init(bar(B_Q_FREE + b), 1);
            mbar_init(bar(B_S_FULL + b), 1);
            mbar_init(bar(B_P_FULL + b), 256);
            mbar_init(bar(B_PV_DONE + b), 1);
            mbar_init(bar(B_STATS_FULL + b), 256);
            mbar_init(bar(B_STATS_EMPTY + b), 128);
        }
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(bar(B_K_FULL + s), 1);
            mbar_init(bar(B_K_EMPTY + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(bar(B_V_FULL + s), 1);
            mbar_init(bar(B_V_EMPTY + s), 1);
        }
        mbar_init(bar(B_O_FULL), 1);
        mbar_init(bar(B_O_FREE), 128);
        mbar_init(bar(B_DRAIN), 1);
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
    if (tid < kHD) s_wq[tid] = p.q_norm_w[tid];
    if (tid >= 128 && tid < 192) s_inv[tid - 128] = exp2(-(double)(tid - 128) / 64.0 * log2((double)p.rope_theta));
    if (warp == 2) {
        const float mq = warp_max_abs128(p.q_norm_w);
        const float mk = warp_max_abs128(p.k_norm_w);
        if (lane == 0) {
            const int eq = prescale_exponent(mq), ek = prescale_exponent(mk);
            misc->q_scale = ldexpf(1.f, eq);
            misc->logit_scale = ldexpf(1.4426950408889634f * 0.08838834764831845f, -(eq + ek));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const int n_units = hdr->n_items * kHKV;

    if (warp < 4) {
      regs_dec<kRegsControl>();
      if (warp == 0) {
        // ============================================================ scheduler, K producer
        if (lane == 0) {
            SchedCursor sc;
            uint32_t kst = 0, kph = 0, narm_k = 0;
            for (;;) {
                int u = atomicAdd(&hdr->counter, 1);
                if (u >= n_units) u = -1;
                if (!mbar_wait(bar(B_SCHED_EMPTY + sc.slot), sc.phase ^ 1, abort_flag, status)) break;
                misc->sched[sc.slot] = u;
                mbar_arrive(bar(B_SCHED_FULL + sc.slot));
                sc.advance();
                if (u < 0) break;
                const ItemView it = load_item(items, u, p.window);
                bool ok = true;
                for (int c = 0; c < it.nch && ok; ++c) {
                    ok = mbar_wait(bar(B_K_EMPTY + kst), kph ^ 1, abort_flag, status);
                    if (!ok) break;
                    const uint32_t dst = sbase + kOffK + kst * kTileBytes;
                    const int ks = it.kb + kKeyChunk * c;
                    mbar_expect_tx(bar(B_K_FULL + kst), kTileBytes);
                    tma_load_3d(dst, &tm_k, bar(B_K_FULL + kst), 0, it.g, ks);
                    tma_load_3d(dst + kHalfTile, &tm_k, bar(B_K_FULL + kst), 64, it.g, ks);
                    ++narm_k;
                    if (++kst == kKStages) { kst = 0; kph ^= 1; }
                }
                if (!ok) break;
            }
            // drain: every armed load has landed before shared memory is released
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            volatile int never = 0;
            for (uint32_t s = 0; s < (uint32_t)kKStages; ++s) {
                // stage s received loads number s, s+3, s+6, ...
                const uint32_t nk = narm_k > s ? (narm_k - s + kKStages - 1) / kKStages : 0;
                if (nk) mbar_wait(bar(B_K_FULL + s), (nk - 1) & 1, &never, nullptr, lim);
            }
        }
      } else if (warp == 3) {
        // ============================================================ Q producer
        // Raw Q tiles run ahead of the K stream: the next item's tile is
        // loaded as soon as the tile warpgroup has read the current one.
        if (lane == 0) {
            SchedCursor sc;
            uint32_t n = 0;
            for (;;) {
                if (!mbar_wait(bar(B_SCHED_FULL + sc.slot), sc.phase, abort_flag, status)) break;
                const int u = misc->sched[sc.slot];
                mbar_arrive(bar(B_SCHED_EMPTY + sc.slot));
                sc.advance();
                if (u < 0) break;
                const ItemView it = load_item(items, u, p.window);
                if (!mbar_wait(bar(B_QRAW_EMPTY), (n & 1) ^ 1, abort_flag, status)) break;
                mbar_expect_tx(bar(B_QRAW_FULL), kTileBytes);
                tma_load_3d(sbase + kOffQraw, &tm_q, bar(B_QRAW_FULL), 0, kGroup * it.g, it.q0);
                tma_load_3d(sbase + kOffQraw + kHalfTile, &tm_q, bar(B_QRAW_FULL), 64, kGroup * it.g, it.q0);
                ++n;
            }
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            volatile int never = 0;
            if (n) mbar_wait(bar(B_QRAW_FULL), (n - 1) & 1, &never, nullptr, lim);
        }
      } else if (warp == 2) {
        // ============================================================ V producer
        if (lane == 0) {
            SchedCursor sc;
            uint32_t vst = 0, vph = 0, narm_v = 0;
            for (;;) {
                if (!mbar_wait(bar(B_SCHED_FULL + sc.slot), sc.phase, abort_flag, status)) break;
                const int u = misc->sched[sc.slot];
                mbar_arrive(bar(B_SCHED_EMPTY + sc.slot));
                sc.advance();
                if (u < 0) break;
                const ItemView it = load_item(items, u, p.window);
                bool ok = true;
                for (int c = 0; c < it.nch && ok; ++c) {
                    ok = mbar_wait(bar(B_V_EMPTY + vst), vph ^ 1, abort_flag, status);
                    if (!ok) break;
                    const uint32_t dst = sbase + kOffV + vst * kTileBytes;
                    const int ks = it.kb + kKeyChunk * c;
                    mbar_expect_tx(bar(B_V_FULL + vst), kTileBytes);
                    tma_load_3d(dst, &tm_v, bar(B_V_FULL + vst), 0, it.g, ks);
                    tma_load_3d(dst + kHalfTile, &tm_v, bar(B_V_FULL + vst), 64, it.g, ks);
                    ++narm_v;
                    if (++vst == kVStages) { vst = 0; vph ^= 1; }
                }
                if (!ok) break;
            }
            const unsigned long long lim = 100ull * 1000ull * 1000ull;
            volatile int never = 0;
            for (uint32_t s = 0; s < (uint32_t)kVStages; ++s) {
                const uint32_t nv = narm_v > s ? (narm_v - s + kVStages - 1) / kVStages : 0;
                if (nv) mbar_wait(bar(B_V_FULL + s), (nv - 1) & 1, &never, nullptr, lim);
            }
        }
      } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_f16(1, 1, 1, 128);
            // Descriptor words: only the low word (start address) changes
            // between MMAs, one 32-bit add each.
            const uint64_t dk0 = smem_desc_sw128(sbase + kOffK, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + kOffV, kHalfTile, 1024);
            const uint32_t k_lo = (uint32_t)dk0, k_hi = (uint32_t)(dk0 >> 32);
            const uint32_t v_lo = (uint32_t)dv0, v_hi = (uint32_t)(dv0 >> 32);
            constexpr uint32_t kTileStep = kTileBytes >> 4;
            SchedCursor sc;
            uint32_t kst = 0, kph = 0, vst = 0, vph = 0;
            uint32_t n_fetched = 0, fifo_head = 0, fifo_tail = 0;
            uint32_t s_next = 0;                 // global QK chunk counter
            bool ok = true;
            // fetch the next work unit and append it to the item queue:
            // (kb, ke, nch, item index); nch = -1 marks the end
            auto fetch = [&]() -> int4 {
                int4 e = make_int4(0, 0, -1, 0);
                if (!mbar_wait(bar(B_SCHED_FULL + sc.slot), sc.phase, abort_flag, status)) { ok = false; return e; }
                const int u = misc->sched[sc.slot];
                mbar_arrive(bar(B_SCHED_EMPTY + sc.slot));
                sc.advance();
                if (u >= 0) {
                    const ItemView it = load_item(items, u, p.window);
                    e = make_int4(it.kb, it.ke, it.nch, (int)n_fetched++);
                }
                s_fifo[fifo_tail & 3] = e;
                ++fifo_tail;
                return e;
            };
            int4 qk_item = fetch();
            int qk_c = 0;
            bool qk_live = ok && qk_item.z >= 0;
            // S = Q K^T for the next chunk of the QK cursor (two chunks ahead
            // of the PV cursor); A = normalised Q from TMEM, B = K from smem.
            auto issue_qk = [&]() {
                if (!qk_live || !ok) return;
                if (qk_c == qk_item.z) {
                    qk_item = fetch();
                    qk_c = 0;
                    if (!ok || qk_item.z < 0) { qk_live = false; return; }
                }
                const uint32_t n = (uint32_t)qk_item.w, qb = n & 1;
                if (qk_c == 0) {
                    ok = mbar_wait(bar(B_Q_READY + qb), (n >> 1) & 1, abort_flag, status);
                    if (!ok) return;
                }
                ok = mbar_wait(bar(B_K_FULL + kst), kph, abort_flag, status);
                if (!ok) return;
                tc_fence_after();
                const int ks = qk_item.x + kKeyChunk * qk_c;
                const uint32_t idesc = idesc_f16(0, 0, 0, (uint32_t)chunk_cols(ks, qk_item.y));
                const uint32_t b = s_next & 1;
                const uint32_t d = tmem + kTmemS + 128u * b;
                const uint32_t qa = tmem + kTmemQ + 64u * qb;
                const uint32_t kb_ = k_lo + kst * kTileStep;
#pragma unroll
                for (uint32_t kk = 0; kk < kHD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (kHalfTile >> 4) + (kk & 3) * 2;
                    mma_ts_w(d, qa + 8u * kk, kb_ + off, k_hi, idesc_f16(0, 0, 0, 0) | idesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(B_S_FULL + b));
                mma_commit(bar(B_K_EMPTY + kst));
                if (qk_c == qk_item.z - 1) mma_commit(bar(B_Q_FREE + qb));
                if (++kst == kKStages) { kst = 0; kph ^= 1; }
                ++qk_c;
                ++s_next;
            };
            issue_qk();
            issue_qk();
            uint32_t pv_g = 0, n_pv = 0;
            while (ok) {
                const int4 it = s_fifo[fifo_head & 3];
                ++fifo_head;
                if (it.z < 0) break;
                for (int c = 0; c < it.z && ok; ++c) {
                    const uint32_t b = pv_g & 1;
                    ok = mbar_wait(bar(B_P_FULL + b), (pv_g >> 1) & 1, abort_flag, status);
                    if (!ok) break;
                    if (c == 0 && n_pv > 0) {
                        ok = mbar_wait(bar(B_O_FREE), (n_pv - 1) & 1, abort_flag, status);
                        if (!ok) break;
                    }
                    ok = mbar_wait(bar(B_V_FULL + vst), vph, abort_flag, status);
                    if (!ok) break;
                    tc_fence_after();
                    const int ks = it.x + kKeyChunk * c;
                    const int nk = chunk_cols(ks, it.y) >> 4;
                    const uint32_t vb = v_lo + vst * kTileStep;
                    const uint32_t d = tmem + kTmemO, pa = tmem + kTmemS + 128u * b;
                    mma_ts_w(d, pa, vb, v_hi, idesc_pv, c > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 1; kk < 8; ++kk)
                        if (kk < nk) mma_ts_w(d, pa + 8u * kk, vb + kk * (2048 >> 4), v_hi, idesc_pv, 1u);
                    mma_commit(bar(B_V_EMPTY + vst));
                    mma_commit(bar(B_PV_DONE + b));
                    if (c == it.z - 1) mma_commit(bar(B_O_FULL));
                    if (++vst == kVStages) { vst = 0; vph ^= 1; }
                    ++pv_g;
                    issue_qk();
                }
                ++n_pv;
            }
            // drain: every MMA issued so far has completed
            mma_commit(bar(B_DRAIN));
            volatile int never = 0;
            mbar_wait(bar(B_DRAIN), 0, &never, nullptr, 100ull * 1000ull * 1000ull);
        }
      }
    } else if (warp < 12) {
        regs_inc<kRegsSoftmax>();
        // ============================================================ softmax
        // Two warpgroups share every row: w = 0 takes columns 0-63 of each S
        // chunk, w = 1 columns 64-127.  Their partial row maxima meet in
        // shared memory behind one 256-thread barrier per chunk, which also
        // makes every abort decision common to both.
        const int w = (warp - 4) >> 2;               // column half
        const int r = (tid - 128) & 127;             // row = TMEM lane, 0..127
        const int tl = r >> 3, hl = r & 7;           // token within tile, head within group
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u;
        const uint32_t t_row = tmem + (lane_base << 16);
        const uint32_t t_o = t_row + kTmemO + 64u * w;     // this half's O columns
        const float C = misc->logit_scale;
        SchedCursor sc;
        uint32_t gchunk = 0, n = 0;
        // `good` is warp-uniform; every exit goes through a 256-thread AND so
        // both warpgroups leave together and no named barrier is left waiting.
        bool good = true;
        for (;;) {
            bool ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SCHED_FULL + sc.slot), sc.phase, abort_flag, status));
            const int u = ok ? misc->sched[sc.slot] : -1;
            good = block_and(1, 256, good && ok);
            if (!good) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SCHED_EMPTY + sc.slot));
            sc.advance();
            if (u < 0) break;
            const ItemView it = load_item(items, u, p.window);
            const int h = kGroup * it.g + hl;
            const int i = it.q0 + tl;
            const float sink = p.sinks[h];
            float m = sink * 1.4426950408889634f;      // log2 domain
            float l = (w == 0 && sink != -INFINITY) ? 1.f : 0.f;   // the sink column counts once
            const int lo = p.window > 0 ? i - p.window + 1 : -(1 << 30);
            for (int c = 0; c < it.nch; ++c, ++gchunk) {
                const int ks = it.kb + kKeyChunk * c;
                const int nc = chunk_cols(ks, it.ke);
                const int mycols = min(max(nc - 64 * w, 0), 64);
                const int nblk = (mycols + 31) >> 5;   // 0, 1 or 2 blocks of 32 columns
                const uint32_t b = gchunk & 1;
                const uint32_t t_s = t_row + kTmemS + 128u * b;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + b), (gchunk >> 1) & 1, abort_flag, status));
                ok = ok && good;
                const bool boundary = (c == it.nch - 1) || (ks + nc - 1 > it.q0) ||
                                      (p.window > 0 && ks < it.q0 + kTokPerTile - p.window);
                uint32_t sv[64];
                float mxp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb)
                        if (bb < nblk) tmem_ld32(t_s + 64u * w + 32u * bb, sv + 32 * bb);
                    tmem_wait_ld();
                    if (boundary) {
                        const int jlo = lo - ks - 64 * w, jhi = i - ks - 64 * w;
#pragma unroll
                        for (int bb = 0; bb < 2; ++bb) {
                            if (bb < nblk) {
#pragma unroll
                                for (int j = 32 * bb; j < 32 * bb + 32; j += 2) {
                                    const float x0 = ((j >= jlo) && (j <= jhi)) ? __uint_as_float(sv[j]) : -INFINITY;
                                    const float x1 = ((j + 1 >= jlo) && (j + 1 <= jhi)) ? __uint_as_float(sv[j + 1]) : -INFINITY;
                                    sv[j] = __float_as_uint(x0);
                                    sv[j + 1] = __float_as_uint(x1);
                                    mxp[(j >> 1) & 3] = max3(mxp[(j >> 1) & 3], x0, x1);
                                }
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; j += 2)
                            mxp[(j >> 1) & 3] = max3(mxp[(j >> 1) & 3], __uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
                    }
                }
                const float pm = fmaxf(max3(mxp[0], mxp[1], mxp[2]), mxp[3]);
                float* px = s_pmax + (b * 2) * 128;
                px[w * 128 + r] = pm;
                good = block_and(1, 256, ok);
                if (!good) break;
                const float mx = fmaxf(pm, px[(1 - w) * 128 + r]);
                // both halves take the same decisions from the same maxima
                const float m_new = fmaxf(m, mx * C);
                const bool raise = (c == 0) ? (m_new > m) : (m_new > m + 8.f);
                float alpha = 1.f;
                if (raise) {
                    alpha = ex2(m - m_new);
                    l *= alpha;
                }
                // rescale this half of O in TMEM once the previous chunk's PV
                // has landed (warp-uniform: tcgen05.ld/st are .sync.aligned)
                if (c > 0 && __any_sync(0xffffffffu, raise)) {
                    const uint32_t pg = gchunk - 1;
                    good = __all_sync(0xffffffffu, mbar_wait(bar(B_PV_DONE + (pg & 1)), (pg >> 1) & 1, abort_flag, status));
                    if (!good) continue;     // leaves at the next 256-thread AND
                    tc_fence_after();
#pragma unroll 1
                    for (int bb = 0; bb < 4; ++bb) {
                        uint32_t v[16];
                        tmem_ld16(t_o + 16u * bb, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
                        tmem_st16(t_o + 16u * bb, v);
                    }
                }
                if (raise) m = m_new;
                const float negm = (m == -INFINITY) ? 0.f : -m;
                const uint64_t C2 = f2(C, C), negm2 = f2(negm, negm);
                uint64_t lp[4];
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) lp[k4] = 0ull;   // (+0.0f, +0.0f)
                // Part of the pairs of an unmasked chunk go through the
                // polynomial; masked chunks and infinite maxima keep ex2 so
                // -inf maps to exactly 0.  P of key k goes to column k/2.
                const uint32_t t_p = t_s + 32u * w;
                const bool use_poly =
                    __all_sync(0xffffffffu, !boundary && m > -INFINITY && m < INFINITY);
                if (use_poly) {
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint64_t x = f2_fma(f2(__uint_as_float(sv[32 * bb + 2 * j]),
                                                         __uint_as_float(sv[32 * bb + 2 * j + 1])), C2, negm2);
                            uint64_t pp;
                            if ((j & 7) < kPolyPairs) pp = exp2_poly2(x);
                            else pp = f2(ex2(f2_lo(x)), ex2(f2_hi(x)));
                            lp[j & 3] = f2_add(lp[j & 3], pp);
                            pk[j] = pack_bf16(f2_lo(pp), f2_hi(pp));
                        }
                        tmem_st16(t_p + 16u * bb, pk);
                    }
                } else {
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        if (bb < nblk) {
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const uint64_t x = f2_fma(f2(__uint_as_float(sv[32 * bb + 2 * j]),
                                                             __uint_as_float(sv[32 * bb + 2 * j + 1])), C2, negm2);
                                const uint64_t pp = f2(ex2(f2_lo(x)), ex2(f2_hi(x)));
                                lp[j & 3] = f2_add(lp[j & 3], pp);
                                pk[j] = pack_bf16(f2_lo(pp), f2_hi(pp));
                            }
                            tmem_st16(t_p + 16u * bb, pk);
                        }
                    }
                }
                const uint64_t ls = f2_add(f2_add(lp[0], lp[1]), f2_add(lp[2], lp[3]));
                l += f2_lo(ls) + f2_hi(ls);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P_FULL + b));
            }
            good = block_and(1, 256, good);
            if (!good) break;
            // final (m, partial l) of this item's rows for the epilogue
            good = __all_sync(0xffffffffu, mbar_wait(bar(B_STATS_EMPTY + (n & 1)), ((n >> 1) & 1) ^ 1, abort_flag, status));
            if (!good) continue;             // leaves at the next 256-thread AND
            float* st = reinterpret_cast<float*>(s_stats + (n & 1) * 128 + r);
            if (w == 0) { st[0] = m; st[1] = l; } else { st[2] = l; }
            mbar_arrive(bar(B_STATS_FULL + (n & 1)));
            ++n;
        }
    } else {
        regs_dec<kRegsTile>();
        // ============================================================ tile warpgroup:
        // Q prologue of the next item, epilogue of the previous one
        const int r = tid - 384;                     // row = TMEM lane, 0..127
        const int tl = r >> 3, hl = r & 7;
        const uint32_t lane_base = (uint32_t)(warp & 3) * 32u;
        const uint32_t t_row = tmem + (lane_base << 16);
        const uint8_t* qraw = smem + kOffQraw;
        float2* rope_tab = reinterpret_cast<float2*>(smem + kOffRope);
        const float qs = misc->q_scale;
        SchedCursor sc;
        uint32_t n = 0;
        int4 prev = make_int4(0, 0, 0, 0);   // (q0, nq, g, valid) of the item awaiting its epilogue
        auto epilogue = [&](const int4 e, uint32_t j) -> bool {
            bool ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), j & 1, abort_flag, status));
            if (!ok) return false;
            tc_fence_after();
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_STATS_FULL + (j & 1)), (j >> 1) & 1, abort_flag, status));
            if (!ok) return false;
            const float4 st = s_stats[(j & 1) * 128 + r];
            mbar_arrive(bar(B_STATS_EMPTY + (j & 1)));
            const float m = st.x, l = st.y + st.z;
            const int i = e.x + tl;
            const int h = kGroup * e.z + hl;
            const bool row_valid = tl < e.y;
            const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
            __nv_bfloat16* orow = p.out + ((size_t)i * kHQ + h) * kHD;
            uint32_t v[64];
            tmem_ld32(t_row + kTmemO, v);
            tmem_ld32(t_row + kTmemO + 32u, v + 32);
            tmem_wait_ld();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (half == 1) {
                    tmem_ld32(t_row + kTmemO + 64u, v);
                    tmem_ld32(t_row + kTmemO + 96u, v + 32);
                    tmem_wait_ld();
                }
                if (half == 1) {
                    // every read of O is done: release it for the next item's PV
                    tc_fence_before();
                    mbar_arrive(bar(B_O_FREE));
                }
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + 64 * half);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_uint4(pack_bf16(__uint_as_float(v[8 * j + 0]) * inv_l, __uint_as_float(v[8 * j + 1]) * inv_l),
                                            pack_bf16(__uint_as_float(v[8 * j + 2]) * inv_l, __uint_as_float(v[8 * j + 3]) * inv_l),
                                            pack_bf16(__uint_as_float(v[8 * j + 4]) * inv_l, __uint_as_float(v[8 * j + 5]) * inv_l),
                                            pack_bf16(__uint_as_float(v[8 * j + 6]) * inv_l, __uint_as_float(v[8 * j + 7]) * inv_l));
                }
            }
            if (row_valid && p.lse) p.lse[(size_t)h * p.T + i] = m * 0.6931471805599453f + logf(l);
            return true;
        };
        for (;;) {
            bool ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SCHED_FULL + sc.slot), sc.phase, abort_flag, status));
            if (!ok) break;
            const int u = misc->sched[sc.slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SCHED_EMPTY + sc.slot));
            sc.advance();
            if (u < 0) break;
            const ItemView it = load_item(items, u, p.window);
            const int i = it.q0 + tl;
            // ---- rope table for this item's 16 tokens: thread r fills token
            // tl, pair indices 8*hl .. 8*hl+7.  The 8 threads of a token are
            // lanes of one warp, so a warp barrier publishes the entries.
            __syncwarp();
            if (p.use_rope) {
                const int tok = min(i, p.T - 1);
                const int pos = p.pos_ids ? p.pos_ids[tok] : (i - it.ds);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float c, s;
                    rope_cos_sin(pos, s_inv[8 * hl + e], &c, &s);
                    rope_tab[tl * 64 + 8 * hl + e] = make_float2(c, s);
                }
            }
            __syncwarp();
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_QRAW_FULL), n & 1, abort_flag, status));
            if (!ok) break;
            // ---- Q prologue: RMSNorm (weight form), RoPE, x 2^eq, FP16, into
            // TMEM.  Thread r owns row r; chunk c of each 64-channel half of
            // the raw tile sits at the 128-byte-swizzled position (c ^ (r & 7)).
            uint32_t qw[64];                     // column j holds channels 2j, 2j+1
            {
                const int sw = r & 7;
                float ss = 0.f;
#pragma unroll 2
                for (int c = 0; c < 8; ++c) {
                    const int off = r * 128 + ((c ^ sw) << 4);
                    const uint4 ua = *reinterpret_cast<const uint4*>(qraw + off);
                    const uint4 ub = *reinterpret_cast<const uint4*>(qraw + kHalfTile + off);
                    const uint32_t w8[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float x0 = bf16_lo(w8[j]), x1 = bf16_hi(w8[j]);
                        ss = fmaf(x0, x0, ss);
                        ss = fmaf(x1, x1, ss);
                    }
                }
                const float rn = rsqrtf(ss * (1.f / kHD) + p.eps) * qs;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int off = r * 128 + ((c ^ sw) << 4);
                    const uint4 ua = *reinterpret_cast<const uint4*>(qraw + off);
                    const uint4 ub = *reinterpret_cast<const uint4*>(qraw + kHalfTile + off);
                    const uint32_t wa4[4] = {ua.x, ua.y, ua.z, ua.w};
                    const uint32_t wb4[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int d0 = 8 * c + 2 * e;          // channels d0, d0+1 and 64+d0, 65+d0
                        float a0 = bf16_lo(wa4[e]) * rn * s_wq[d0];
                        float a1 = bf16_hi(wa4[e]) * rn * s_wq[d0 + 1];
                        float b0 = bf16_lo(wb4[e]) * rn * s_wq[64 + d0];
                        float b1 = bf16_hi(wb4[e]) * rn * s_wq[65 + d0];
                        if (p.use_rope) {
                            const float2 cs0 = rope_tab[tl * 64 + d0];
                            const float2 cs1 = rope_tab[tl * 64 + d0 + 1];
                            const float y0 = a0 * cs0.x - b0 * cs0.y, z0 = b0 * cs0.x + a0 * cs0.y;
                            const float y1 = a1 * cs1.x - b1 * cs1.y, z1 = b1 * cs1.x + a1 * cs1.y;
                            a0 = y0; b0 = z0; a1 = y1; b1 = z1;
                        }
                        qw[4 * c + e] = pack_f16(a0, a1);
                        qw[32 + 4 * c + e] = pack_f16(b0, b1);
                    }
                }
            }
            // the raw tile has been read: let the producer load the next one
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_QRAW_EMPTY));
            const uint32_t qb = n & 1;
            if (n >= 2) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_Q_FREE + qb), ((n - 2) >> 1) & 1, abort_flag, status));
                if (!ok) break;
                tc_fence_after();
            }
            tmem_st32(t_row + kTmemQ + 64u * qb, qw);
            tmem_st32(t_row + kTmemQ + 64u * qb + 32u, qw + 32);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_Q_READY + qb));
            // ---- epilogue of the previous item
            if (n >= 1 && !epilogue(prev, n - 1)) break;
            prev = make_int4(it.q0, it.nq, it.g, 1);
            ++n;
        }
        if (n >= 1 && prev.w) epilogue(prev, n - 1);
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

extern const unsigned kAttnSmemBytes = kSmemBytes;
extern const unsigned kAttnThreads = kThreads;

}  // namespace flint
