// Preparation kernel of the Flint attention forward.
//
// Block 0 builds the work plan: it reads the document boundaries (packed THD
// cu_seqlens) or the per-row valid lengths of a trailing padding mask,
// splits every document into work items of 32 tokens and orders the items by
// their number of 128-key chunks, longest first, so the attention kernel's
// dynamic scheduler hands out the largest items first.
//
// The other blocks prepare the keys once per token instead of once per use
// (each key is read by up to 33 query tiles on a sliding layer): per-head
// RMSNorm with k_norm_w (weight form; HF discussion #26 on RecursiveSI/flint),
// then on sliding layers NeoX RoPE at the document-local position
// (FlintAttention._apply_rope), scaled by a power of two and rounded to FP16
// into the workspace.  Queries are used by one tile only: on full layers the
// attention kernel normalises and rotates them itself; on sliding layers
// (units of ~5 chunks, too short to hide that prologue) these blocks do it,
// into the token's own output rows as FP16, and on calls of at most 2,048
// tokens they spread each token over nine warps.  Padded query tokens get
// their final outputs here: zeros and lse = sink (FlintAttention.forward,
// attention_mask: the sink remains valid for padded queries).
#include "flint_common.cuh"
#include "sm100.cuh"

namespace flint {

// ---------------------------------------------------------------- block scan
// Inclusive prefix sum over the 1024 threads of the block; returns the block
// total in *total.  `sh` holds 33 ints.
__device__ int block_incl_scan(int v, int* sh, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? sh[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        sh[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    int r = v + (warp > 0 ? sh[warp - 1] : 0);
    *total = sh[(blockDim.x >> 5) - 1];
    __syncthreads();
    return r;
}

// Last segment s with prefix[s] <= it (prefix non-decreasing, prefix[0] = 0).
__device__ __forceinline__ int find_segment(const int* prefix, int nseg, int it) {
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= it) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct ItemDesc { int q0, nq, ds, nch; };

__device__ __forceinline__ ItemDesc describe_item(const int2* seg, const int* prefix, int nseg,
                                                 int it, int window) {
    int s = find_segment(prefix, nseg, it);
    // skip empty segments that share the same prefix value
    while (s + 1 < nseg && prefix[s + 1] <= it) ++s;
    int li = it - prefix[s];
    int2 sg = seg[s];
    ItemDesc d;
    d.ds = sg.x;
    d.q0 = sg.x + kTokPerItem * li;
    d.nq = min(kTokPerItem, sg.y - kTokPerItem * li);
    int ke = d.q0 + d.nq;
    int kb = window > 0 ? max(d.ds, d.q0 - window + 1) : d.ds;
    d.nch = (ke - kb + kKeyChunk - 1) / kKeyChunk;
    return d;
}

__device__ void build_plan(const PrepParams& p) {
    __shared__ int sh[33];
    __shared__ int s_status;
    const WsLayout L = ws_layout(p.T, p.nseg);
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(p.ws + L.header);
    int2* seg = reinterpret_cast<int2*>(p.ws + L.seg);
    int* prefix = reinterpret_cast<int*>(p.ws + L.prefix);
    int* hist = reinterpret_cast<int*>(p.ws + L.hist);
    int4* items = reinterpret_cast<int4*>(p.ws + L.items);
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarp = nthr >> 5;

    if (tid == 0) s_status = kStatusOk;
    for (int i = tid; i < L.hist_len; i += nthr) hist[i] = 0;
    __syncthreads();

    // 1. segments (start, valid length)
    if (p.mode == kMaskThd) {
        const int* cu = p.cu_seqlens;
        if (tid == 0 && (cu[0] != 0 || cu[p.nseg] > p.T || cu[p.nseg] < 0))
            atomicExch(&s_status, kStatusInvalid);
        for (int s = tid; s < p.nseg; s += nthr) {
            int a = cu[s], b = cu[s + 1];
            if (b < a || a < 0) atomicExch(&s_status, kStatusInvalid);
            seg[s] = make_int2(a, max(b - a, 0));
        }
    } else if (p.mode == kMaskPad) {
        for (int row = warp; row < p.batch; row += nwarp) {
            const uint8_t* m = p.pad_mask + (size_t)row * p.seqlen;
            int cnt = 0, first_zero = p.seqlen, bad = 0;
            for (int j = lane; j < p.seqlen; j += 32) {
                int v = m[j];
                if (v == 1) ++cnt;
                else if (v == 0) first_zero = min(first_zero, j);
                else bad = 1;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
                first_zero = min(first_zero, __shfl_xor_sync(0xffffffffu, first_zero, o));
                bad |= __shfl_xor_sync(0xffffffffu, bad, o);
            }
            if (lane == 0) {
                if (bad) atomicExch(&s_status, kStatusInvalid);
                else if (first_zero < cnt) atomicCAS(&s_status, kStatusOk, kStatusUnsupported);
                seg[row] = make_int2(row * p.seqlen, cnt);
            }
        }
    } else {
        if (tid == 0) seg[0] = make_int2(0, p.T);
    }
    __syncthreads();

    // 2. items per segment, exclusive prefix over segments
    int running = 0;
    for (int base = 0; base < p.nseg; base += nthr) {
        int s = base + tid;
        int n = 0;
        if (s < p.nseg) n = (seg[s].y + kTokPerItem - 1) / kTokPerItem;
        int tot;
        int incl = block_incl_scan(n, sh, &tot);
        if (s < p.nseg) prefix[s] = running + incl - n;
        running += tot;
    }
    if (tid == 0) prefix[p.nseg] = running;
    const int n_items = (s_status == kStatusOk) ? running : 0;
    __syncthreads();

    // 3. histogram of chunk counts
    for (int it = tid; it < n_items; it += nthr) {
        ItemDesc d = describe_item(seg, prefix, p.nseg, it, p.window);
        atomicAdd(&hist[d.nch], 1);
    }
    __syncthreads();

    // 4. descending exclusive offsets: bin c starts after all bins c' > c
    running = 0;
    for (int base = 0; base < L.hist_len; base += nthr) {
        int rb = base + tid;                       // reversed bin index
        int c = L.hist_len - 1 - rb;
        int n = (rb < L.hist_len) ? hist[c] : 0;
        int tot;
        int incl = block_incl_scan(n, sh, &tot);
        if (rb < L.hist_len) hist[c] = running + incl - n;
        running += tot;
    }
    __syncthreads();

    // 5. scatter
    for (int it = tid; it < n_items; it += nthr) {
        ItemDesc d = describe_item(seg, prefix, p.nseg, it, p.window);
        int at = atomicAdd(&hist[d.nch], 1);
        items[at] = make_int4(d.q0, d.nq, d.ds, d.nch);
    }
    __syncthreads();
    if (tid == 0) {
        hdr->status = s_status;
        hdr->n_items = n_items;
        hdr->counter = 0;
    }
}

// ---------------------------------------------------------------- key prep

__device__ __forceinline__ int thd_segment_start(const int* cu, int ndocs, int t) {
    // last d with cu[d] <= t
    int lo = 0, hi = ndocs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return cu[lo];
}

// Normalise one 128-channel head row held by 8 lanes (lane sub owns channels
// 8*sub .. 8*sub+7 of each 64-channel half): RMSNorm in weight form, optional
// NeoX rotation with the lane's 8 (cos, sin) pairs, x scale, FP16.
// The lane's 16 input values: channels 8 sub .. 8 sub + 7 and 64 + 8 sub ..
__device__ __forceinline__ void load_row16(const __nv_bfloat16* src, int sub, float* x0, float* x1) {
    const uint4 a = *reinterpret_cast<const uint4*>(src + 8 * sub);
    const uint4 b = *reinterpret_cast<const uint4*>(src + 64 + 8 * sub);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(pa[e]);
        const float2 fb = __bfloat1622float2(pb[e]);
        x0[2 * e] = fa.x; x0[2 * e + 1] = fa.y;
        x1[2 * e] = fb.x; x1[2 * e + 1] = fb.y;
    }
}
__device__ __forceinline__ void load_row16(const float* src, int sub, float* x0, float* x1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float4 a = *reinterpret_cast<const float4*>(src + 8 * sub + 4 * h);
        const float4 b = *reinterpret_cast<const float4*>(src + 64 + 8 * sub + 4 * h);
        x0[4 * h] = a.x; x0[4 * h + 1] = a.y; x0[4 * h + 2] = a.z; x0[4 * h + 3] = a.w;
        x1[4 * h] = b.x; x1[4 * h + 1] = b.y; x1[4 * h + 2] = b.z; x1[4 * h + 3] = b.w;
    }
}

template <typename In>
__device__ __forceinline__ void norm_rope_row(const In* src, __half* dst, const float* w,
                                              float eps, float scale, int sub, bool rope,
                                              const float* cc, const float* sn, bool store = true) {
    float x0[8], x1[8];
    load_row16(src, sub, x0, x1);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(x0[e], x0[e], fmaf(x1[e], x1[e], ss));
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    const float r = rsqrtf(ss * (1.f / kHD) + eps) * scale;
    float n0[8], n1[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        n0[e] = x0[e] * r * w[8 * sub + e];
        n1[e] = x1[e] * r * w[64 + 8 * sub + e];
    }
    if (rope) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float y0 = n0[e] * cc[e] - n1[e] * sn[e];
            const float y1 = n1[e] * cc[e] + n0[e] * sn[e];
            n0[e] = y0; n1[e] = y1;
        }
    }
    uint4 oa, ob;
    {
        __half2* ha = reinterpret_cast<__half2*>(&oa);
        __half2* hb = reinterpret_cast<__half2*>(&ob);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            ha[e] = __floats2half2_rn(n0[2 * e], n0[2 * e + 1]);
            hb[e] = __floats2half2_rn(n1[2 * e], n1[2 * e + 1]);
        }
    }
    if (store) {
        *reinterpret_cast<uint4*>(dst + 8 * sub) = oa;
        *reinterpret_cast<uint4*>(dst + 64 + 8 * sub) = ob;
    }
}

// kSplit: the call spreads each token over prep_parts() warps (small calls
// that prepare queries); otherwise one warp takes each token.
template <bool kSplit>
__device__ void prepare_tokens(const PrepParams& p) {
    __shared__ double s_inv_freq[64];
    __shared__ float s_wk[kHD], s_wq[kHD];
    __shared__ float s_kscale, s_qscale;
    __shared__ int s_thd_end;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const WsLayout L = ws_layout(p.T, p.nseg);
    __half* kn = reinterpret_cast<__half*>(p.ws + L.kn);

    if (tid < 64) s_inv_freq[tid] = exp2(-(double)tid / 64.0 * log2((double)p.rope_theta));
    if (tid < kHD) s_wk[tid] = p.k_norm_w[tid];
    if (tid >= kHD && tid < 2 * kHD) s_wq[tid - kHD] = p.q_norm_w[tid - kHD];
    if (warp == 0) {
        const float m = warp_max_abs128(p.k_norm_w);
        if (lane == 0) s_kscale = ldexpf(1.f, prescale_exponent(m));
    }
    if (warp == 1) {
        const float m = warp_max_abs128(p.q_norm_w);
        if (lane == 0) s_qscale = ldexpf(1.f, prescale_exponent(m));
    }
    if (tid == 0) s_thd_end = (p.mode == kMaskThd) ? p.cu_seqlens[p.nseg] : p.T;
    __syncthreads();

    const int head = lane >> 3, sub = lane & 7;
    const int nwarps_total = (gridDim.x - 1) * (blockDim.x >> 5);
    const float kscale = s_kscale;
    const bool rope = p.use_rope != 0;
    // A call of few tokens that also prepares queries spreads each token over
    // 1 + 8 warps (its keys, then its query heads four at a time), so that
    // enough loads are in flight; otherwise one warp takes a token, and its
    // RoPE table serves all of the token's heads.
    const int nparts = kSplit ? prep_parts(p.T, true) : 1;
    const int nwork = p.T * nparts;               // at most 2,048 x 9, or T
    for (int wi = (blockIdx.x - 1) * (blockDim.x >> 5) + warp; wi < nwork; wi += nwarps_total) {
        const int t = kSplit ? wi / nparts : wi, part = kSplit ? wi - t * nparts : 0;
        // query passes hq0 .. hq1 - 1 of this warp (4 heads each); the keys
        // and the padded-row outputs go with part 0
        const int hq0 = kSplit ? (part > 0 ? part - 1 : 0) : 0, hq1 = kSplit ? part : kHQ / kHKV;
        // ---- the lane's 8 (cos, sin) pairs f = 8*sub + e at the token's
        // document-local position, shared by its 4 key heads
        float cc[8], sn[8];
        if (rope && (p.f16 || p.qprep || (!p.keys_ready && part == 0))) {
            int pos;
            if (p.pos_ids) pos = p.pos_ids[t];
            else if (p.mode == kMaskThd) pos = t - (t < s_thd_end ? thd_segment_start(p.cu_seqlens, p.nseg, t) : s_thd_end);
            else if (p.mode == kMaskPad) pos = t % p.seqlen;
            else pos = t;
            // lane computes the pairs 2*lane and 2*lane + 1
            float c0, s0, c1, s1;
            rope_cos_sin(pos, s_inv_freq[2 * lane], &c0, &s0);
            rope_cos_sin(pos, s_inv_freq[2 * lane + 1], &c1, &s1);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int f = 8 * sub + e;
                // (e & 1) is uniform across the warp for a given e, so the
                // selected register is the same in every lane
                cc[e] = __shfl_sync(0xffffffffu, (e & 1) ? c1 : c0, f >> 1);
                sn[e] = __shfl_sync(0xffffffffu, (e & 1) ? s1 : s0, f >> 1);
            }
        }
        // ---- the key heads (head = lane / 8; ng of them, 4 unless the call
        // covers a head slice).  Every lane takes part in the row's shuffles;
        // lanes past the slice normalise a valid row and store nothing.
        const bool kstore = head < p.ng;
        const size_t krow = ((size_t)t * p.ng + (kstore ? head : 0)) * kHD;
        if (part == 0 && p.f16)
            norm_rope_row(p.kf + krow, kn + krow, s_wk, p.eps, kscale, sub, rope, cc, sn, kstore);
        else if (part == 0 && !p.keys_ready)
            norm_rope_row(p.k + krow, kn + krow, s_wk, p.eps, kscale, sub, rope, cc, sn, kstore);
        if (part == 0 && p.f16) {
            // FP16 policy: the values cast to FP16 (4 heads x 128 per token,
            // 16 per lane)
            __half* vh = reinterpret_cast<__half*>(p.ws + L.vh) + (size_t)t * kHKV * kHD;
            const float* vs = p.vf + (size_t)t * kHKV * kHD;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 a = *reinterpret_cast<const float4*>(vs + 4 * lane + 128 * i);
                const __half2 lo = __floats2half2_rn(a.x, a.y), hi = __floats2half2_rn(a.z, a.w);
                *reinterpret_cast<uint2*>(vh + 4 * lane + 128 * i) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
            }
        }

        bool padded;
        if (p.mode == kMaskThd) padded = t >= s_thd_end;
        else if (p.mode == kMaskPad) padded = p.pad_mask[t] == 0;
        else padded = false;
        if (padded) {
            if (part != 0) continue;
            // ---- padded query token: zero output row, lse = sink
            uint4 z = make_uint4(0, 0, 0, 0);
            const int nh = kGroup * p.ng;                  // query heads in the tensors
            uint4* o = reinterpret_cast<uint4*>(p.out + (size_t)t * nh * kHD);
#pragma unroll 4
            for (int i = lane; i < nh * kHD / 8; i += 32) o[i] = z;
            if (p.lse && lane < nh) p.lse[(size_t)lane * p.T + t] = p.sinks[lane];
        } else if (p.f16) {
            // ---- FP16 policy: the 32 query heads normalised and rotated in
            // FP32 and cast to FP16 (x 2^eq) into the workspace, 4 per pass
            const float* qrow = p.qf + (size_t)t * kHQ * kHD;
            __half* qdst = reinterpret_cast<__half*>(p.ws + L.qn) + (size_t)t * kHQ * kHD;
#pragma unroll 2
            for (int hq = hq0; hq < hq1; ++hq) {
                const int hh = kHKV * hq + head;
                norm_rope_row(qrow + hh * kHD, qdst + hh * kHD, s_wq, p.eps, s_qscale, sub, rope, cc, sn);
            }
        } else if (p.qprep) {
            // ---- the query heads (8 ng of them) normalised and rotated into
            // the output rows of the token as FP16 (x 2^eq), 4 per pass: the
            // attention tile that owns the rows reads them back as its Q
            // operand and writes its result over them.  Each head row is read
            // before it is written, so out may be q itself.
            const int nh = kGroup * p.ng;
            const __nv_bfloat16* qrow = p.q + (size_t)t * nh * kHD;
            __half* qdst = reinterpret_cast<__half*>(p.out + (size_t)t * nh * kHD);
#pragma unroll 2
            for (int hq = hq0; hq < hq1; ++hq) {
                const int hh = kHKV * hq + head;
                const bool qstore = hh < nh;
                const int hs = qstore ? hh : 0;
                norm_rope_row(qrow + hs * kHD, qdst + hs * kHD, s_wq, p.eps, s_qscale, sub, rope, cc, sn, qstore);
            }
        }
    }
}

template <bool kSplit>
__global__ void __launch_bounds__(1024, 1) prep_kernel(PrepParams p) {
    // The attention kernel may be scheduled as soon as every block of this
    // grid has started (it is launched as a programmatic dependent and waits
    // for this grid's completion before it reads anything written here).
    // Blocks trigger on entry, so by the time the attention kernel can take
    // an SM, no block of this grid is still waiting for one.
    griddep_launch_dependents();
    if (blockIdx.x == 0) build_plan(p);
    else prepare_tokens<kSplit>(p);
}
template __global__ void prep_kernel<false>(PrepParams);
template __global__ void prep_kernel<true>(PrepParams);

}  // namespace flint
