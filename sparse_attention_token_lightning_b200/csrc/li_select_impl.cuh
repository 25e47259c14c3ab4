// Device code of the top-k selection, included by li_select.cu once per CTA size: the includer
// defines kThreads (threads per CTA, one CTA per query row) before including this file, and
// Params. Everything here is specialised on kThreads.
constexpr int kDigits = 256;



__device__ __forceinline__ uint32_t score_key(float v) {
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

constexpr int kBinCap = 128;          // largest bucket the per-bucket insertion sort takes
constexpr int kBucketsMax = 4096;     // a power of two
// buckets per row: at most kBucketsMax and at most 16 per thread (the largest bucket scan)
constexpr int kNbMax = kBucketsMax < 16 * kThreads ? kBucketsMax : 16 * kThreads;
static_assert(kNbMax % kThreads == 0 && kNbMax / kThreads <= 16, "bucket scan covers 16 per thread");

struct Smem {
    int32_t hist[kDigits];
    int32_t wsum[2][kWarps];
    int32_t s_digit, s_rem, s_cnt;
    int32_t s_skip[4];      // one flag per sort pass, so no pass resets a flag still being read
    float red_min[kWarps], red_max[kWarps];
    float s_vmin, s_vmax;
    int32_t s_cut, s_maxbin;
    int32_t s_append;       // candidate append counter of the long-row path (only used there)
    uint32_t *dbg;          // bounds-checked build: the status word (set at kernel start)
};

// Block-wide exclusive scan of cnt[0..kWarps*kDigits) in place (8 entries per thread).
__device__ void block_exclusive_scan_4096(int32_t *cnt, Smem &sm) {
    constexpr int per = kWarps * kDigits / kThreads;   // 8
    const int tid = threadIdx.x;
    int32_t v[per];
    int32_t local = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) { v[i] = cnt[tid * per + i]; local += v[i]; }
    // warp inclusive scan of local
    const int lane = tid & 31, warp = tid >> 5;
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sm.wsum[0][warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t x = lane < kWarps ? sm.wsum[0][lane] : 0;
        int32_t xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += t;
        }
        if (lane < kWarps) sm.wsum[1][lane] = xi - x;
    }
    __syncthreads();
    int32_t run = sm.wsum[1][warp] + incl - local;
#pragma unroll
    for (int i = 0; i < per; ++i) { cnt[tid * per + i] = run; run += v[i]; }
    __syncthreads();
}

template <bool kCached>
__device__ __forceinline__ uint32_t get_key(const uint32_t *rowc, const float *src, int32_t e) {
    if (kCached) return rowc[e];
    return score_key(__ldcg(src + e));
}

// Radix select: the m-th largest key of n. Leaves (prefix, mask, need) such that the selected
// set is {keys with (u & mask) > prefix} plus the first `need` keys (by index) with
// (u & mask) == prefix.
template <bool kCached>
__device__ void radix_select(const uint32_t *rowc, const float *src, int32_t n, int32_t m,
                             Smem &sm, uint32_t &prefix, uint32_t &mask, int32_t &need) {
    const int tid = threadIdx.x, lane = tid & 31;
    prefix = 0u;
    mask = 0u;
    int32_t rem = m;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < kDigits; i += kThreads) sm.hist[i] = 0;
        __syncthreads();
        for (int32_t e0 = 0; e0 < n; e0 += kThreads) {
            const int32_t e = e0 + tid;
            uint32_t d = kDigits;   // no digit
            if (e < n) {
                const uint32_t u = get_key<kCached>(rowc, src, e);
                if ((u & mask) == prefix) d = (u >> shift) & 0xffu;
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            if (d < kDigits && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[d], __popc(peers));
        }
        __syncthreads();
        if (tid < 32) {
            constexpr int per = kDigits / 32;
            int32_t local = 0;
#pragma unroll
            for (int i = 0; i < per; ++i) local += sm.hist[lane * per + i];
            int32_t incl = local;   // suffix sum over lanes >= this one
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t t = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += t;
            }
            int32_t above = incl - local;
            for (int i = per - 1; i >= 0; --i) {
                const int d = lane * per + i;
                const int32_t c = sm.hist[d];
                if (above < rem && rem <= above + c) {
                    sm.s_digit = d;
                    sm.s_rem = rem - above;
                    sm.s_cnt = c;
                }
                above += c;
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sm.s_digit << shift;
        mask |= 0xffu << shift;
        rem = sm.s_rem;
        const int32_t cnt = sm.s_cnt;
        __syncthreads();
        if (cnt == rem) break;   // every key with this prefix is taken
    }
    need = rem;
}

// Gather the selected keys in index order into keyA/idxA[0..m).
template <bool kCached>
__device__ void gather(const uint32_t *rowc, const float *src, int32_t n, int32_t m,
                       uint32_t prefix, uint32_t mask, int32_t need, uint32_t *keyA,
                       int32_t *idxA, Smem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t gt = m - need;
    int32_t run_gt = 0, run_eq = 0;
    for (int32_t e0 = 0; e0 < n; e0 += kThreads) {
        const int32_t e = e0 + tid;
        uint32_t u = 0;
        bool is_gt = false, is_eq = false;
        if (e < n) {
            u = get_key<kCached>(rowc, src, e);
            const uint32_t mu = u & mask;
            is_gt = mu > prefix;
            is_eq = mu == prefix;
        }
        const uint32_t bg = __ballot_sync(0xffffffffu, is_gt);
        const uint32_t be = __ballot_sync(0xffffffffu, is_eq);
        if (lane == 0) { sm.wsum[0][warp] = __popc(bg); sm.wsum[1][warp] = __popc(be); }
        __syncthreads();
        int32_t pre_g = 0, pre_e = 0, tot_g = 0, tot_e = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int32_t a = sm.wsum[0][w], b = sm.wsum[1][w];
            if (w < warp) { pre_g += a; pre_e += b; }
            tot_g += a;
            tot_e += b;
        }
        const uint32_t lt = lanemask_lt();
        if (is_gt) {
            const int32_t pos = run_gt + pre_g + __popc(bg & lt);
            if (idx_ok(pos, m, sm.dbg)) {
                keyA[pos] = u;
                idxA[pos] = e;
            }
        } else if (is_eq) {
            const int32_t r = run_eq + pre_e + __popc(be & lt);
            if (r < need && idx_ok(gt + r, m, sm.dbg)) {
                keyA[gt + r] = u;
                idxA[gt + r] = e;
            }
        }
        run_gt += tot_g;
        run_eq += tot_e;
        __syncthreads();
    }
}

// Stable LSD radix sort of keyA/idxA[0..m) by key descending. Returns true when the result
// ended in the B buffers.
__device__ bool sort_desc(int32_t m, uint32_t *keyA, int32_t *idxA, uint32_t *keyB, int32_t *idxB,
                          int32_t *cnt, Smem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t seg = (m + kWarps - 1) / kWarps;
    const int32_t s0 = warp * seg, s1 = min(m, s0 + seg);
    bool inB = false;
    if (tid < 4) sm.s_skip[tid] = 0;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 8 * pass;
        uint32_t *ks = inB ? keyB : keyA;
        int32_t *is = inB ? idxB : idxA;
        uint32_t *kd = inB ? keyA : keyB;
        int32_t *id = inB ? idxA : idxB;
        for (int i = tid; i < kWarps * kDigits; i += kThreads) cnt[i] = 0;
        __syncthreads();
        // counts, digit-major: cnt[d * kWarps + w]
        for (int32_t e0 = s0; e0 < s1; e0 += 32) {
            const int32_t e = e0 + lane;
            const uint32_t d = e < s1 ? ((~ks[e]) >> shift) & 0xffu : kDigits;
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            if (d < kDigits && lane == __ffs(peers) - 1) cnt[d * kWarps + warp] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        if (tid < kDigits) {
            int32_t tot = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) tot += cnt[tid * kWarps + w];
            if (tot == m) sm.s_skip[pass] = 1;
        }
        __syncthreads();
        if (sm.s_skip[pass]) continue;   // one digit value for all keys: order unchanged
        block_exclusive_scan_4096(cnt, sm);
        for (int32_t e0 = s0; e0 < s1; e0 += 32) {
            const int32_t e = e0 + lane;
            const bool valid = e < s1;
            const uint32_t key = valid ? ks[e] : 0u;
            const uint32_t d = valid ? ((~key) >> shift) & 0xffu : kDigits;
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            if (valid) {
                const int32_t base = cnt[d * kWarps + warp];
                const int32_t dst = base + __popc(peers & lanemask_lt());
                if (idx_ok(dst, m, sm.dbg)) {
                    kd[dst] = key;
                    id[dst] = is[e];
                }
            }
            __syncwarp();
            if (valid && lane == __ffs(peers) - 1) cnt[d * kWarps + warp] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        inB = !inB;
    }
    return inB;
}

// Bucket of a score: x = (v - vmin) * scale lies in [0, nb]; adding 1.5 * 2^23 leaves round(x)
// in the low mantissa bits (exact for x < 2^22), a monotone integer map without a conversion
// instruction. Bucket 0 holds the highest scores.
__device__ __forceinline__ int32_t bucket_of(float v, float vmin, float scale, int32_t nb) {
    const float x = (v - vmin) * scale;
    int32_t b = __float_as_int(x + 12582912.0f) - 0x4B400000;
    b = b < 0 ? 0 : (b >= nb ? nb - 1 : b);
    return nb - 1 - b;
}

// Block-wide exclusive scan of one value per thread; returns the thread's exclusive prefix. One
// barrier: every warp adds up the totals of the warps before it itself. The caller must pass a
// barrier before sm.wsum is written again.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t x, Smem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sm.wsum[0][warp] = incl;
    __syncthreads();
    int32_t before = lane < warp ? sm.wsum[0][lane] : 0;
#pragma unroll
    for (int o = kWarps / 2; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
    return __shfl_sync(0xffffffffu, before, 0) + incl - x;
}

// Turns the bucket counts into output start positions (exclusive scan in bucket order),
// records the bucket holding output position m-1 in sm.s_cut and the largest count among the
// buckets that start before m in sm.s_maxbin. PER = nb / kThreads buckets per thread. From
// PER = 4 on, warp w owns the 32 PER buckets from 32 PER w on and reads them in steps of 32 int4
// (lane l of step q holds buckets 4 (32 q + l) .. + 3 of the warp's range: consecutive lanes
// read consecutive 16 bytes, no bank conflicts); a warp scan per step and a carry give each
// lane its prefix within the warp, one barrier the warps' prefixes. Below 4, thread t owns
// buckets [PER t, PER (t + 1)).
template <int PER>
__device__ __forceinline__ void scan_buckets(int32_t *hist, int32_t m, Smem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t lmax = 0, cut = -1;
    if constexpr (PER >= 4) {
        constexpr int kSteps = PER / 4;
        int4 *h4 = reinterpret_cast<int4 *>(hist) + warp * 32 * kSteps + lane;
        int32_t pre[kSteps];
        int32_t carry = 0;
#pragma unroll
        for (int q = 0; q < kSteps; ++q) {
            const int4 c = h4[32 * q];
            const int32_t x = c.x + c.y + c.z + c.w;
            int32_t incl = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            pre[q] = carry + incl - x;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) sm.wsum[0][warp] = carry;
        __syncthreads();
        int32_t before = lane < warp ? sm.wsum[0][lane] : 0;
#pragma unroll
        for (int o = kWarps / 2; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
        before = __shfl_sync(0xffffffffu, before, 0);
#pragma unroll
        for (int q = 0; q < kSteps; ++q) {
            const int4 c = h4[32 * q];
            int32_t x[4] = {c.x, c.y, c.z, c.w};
            int32_t run = before + pre[q];
            const int32_t b0 = 4 * ((warp * kSteps + q) * 32 + lane);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int32_t cnt = x[i];
                x[i] = run;
                if (run <= m - 1 && m - 1 < run + cnt) cut = b0 + i;
                if (run < m && cnt > lmax) lmax = cnt;
                run += cnt;
            }
            h4[32 * q] = make_int4(x[0], x[1], x[2], x[3]);
        }
    } else {
        int32_t c[PER];
        if constexpr (PER == 2) {
            const int2 a = reinterpret_cast<const int2 *>(hist)[tid];
            c[0] = a.x; c[1] = a.y;
        } else {
            c[0] = hist[tid];
        }
        int32_t local = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) local += c[i];
        int32_t run = block_exclusive_scan(local, sm);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int32_t x = c[i];
            c[i] = run;
            if (run <= m - 1 && m - 1 < run + x) cut = PER * tid + i;
            if (run < m && x > lmax) lmax = x;
            run += x;
        }
        if constexpr (PER == 2) {
            reinterpret_cast<int2 *>(hist)[tid] = make_int2(c[0], c[1]);
        } else {
            hist[tid] = c[0];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if (lane == 0 && lmax > 0) atomicMax(&sm.s_maxbin, lmax);
    if (cut >= 0) sm.s_cut = cut;
}

constexpr int kRegKeys = 4096 / kThreads;   // keys per thread held in registers (rows <= 4096)
constexpr int kRegQuads = kRegKeys / 4;     // of them, float4 slots
static_assert(kRegKeys % 4 == 0, "register keys come in float4 slots");

// Short-row path (n <= kRegKeys * kThreads): the row is read once with float4 loads (slot i of
// thread tid holds keys 4 (i kThreads + tid) .. + 3) and each key and its bucket stay in
// registers across the passes. Only the first ceil(n / (4 kThreads)) slots are live (a
// block-uniform bound), and only the last of them can reach past the row's end. The row must
// start 16-byte aligned and be readable up to n rounded up to 4 keys: score rows are padded to a
// multiple of 4 floats, and row pieces start at multiples of 128 keys.
// Returns 1 when the stage holds the m output composites in slot order, 3 when all scores tie
// (*vtie set), 2 when the caller must take the exact radix path.
__device__ int reg_bucket_topk(const float *src, int32_t n, int32_t m, int32_t *hist,
                               uint64_t *buf, uint16_t *bufb, uint64_t *stage, Smem &sm,
                               float *vtie) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float kInf = __int_as_float(0x7f800000);
    const int32_t live = (n + 4 * kThreads - 1) / (4 * kThreads);
    int32_t nb = kThreads;
    while (nb < n && nb < kNbMax) nb <<= 1;
    for (int i = tid; i < nb / 4; i += kThreads) reinterpret_cast<int4 *>(hist)[i] = make_int4(0, 0, 0, 0);
    if (tid == 0) { sm.s_cut = nb - 1; sm.s_maxbin = 0; }
    const float4 *src4 = reinterpret_cast<const float4 *>(src);
    float v[kRegKeys];
    float lo = kInf, hi = -kInf;
#pragma unroll
    for (int i = 0; i < kRegQuads; ++i) {
        const int32_t e0 = 4 * (i * kThreads + tid);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < live) {
            if (e0 < n && idx_ok(e0, (n + 3) & ~3, sm.dbg)) x = __ldg(src4 + (e0 >> 2));
            // keys past the row's end leave the minimum and maximum alone (-0 and +0 need no
            // care: they land in the same bucket and have the same composite key)
            lo = fminf(lo, e0 + 0 < n ? x.x : kInf);
            lo = fminf(lo, e0 + 1 < n ? x.y : kInf);
            lo = fminf(lo, e0 + 2 < n ? x.z : kInf);
            lo = fminf(lo, e0 + 3 < n ? x.w : kInf);
            hi = fmaxf(hi, e0 + 0 < n ? x.x : -kInf);
            hi = fmaxf(hi, e0 + 1 < n ? x.y : -kInf);
            hi = fmaxf(hi, e0 + 2 < n ? x.z : -kInf);
            hi = fmaxf(hi, e0 + 3 < n ? x.w : -kInf);
        }
        v[4 * i + 0] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    // one barrier: every warp combines the warps' partial results itself (in the same order, so
    // all warps agree)
    if (lane == 0) { sm.red_min[warp] = lo; sm.red_max[warp] = hi; }
    __syncthreads();
    lo = lane < kWarps ? sm.red_min[lane] : kInf;
    hi = lane < kWarps ? sm.red_max[lane] : -kInf;
#pragma unroll
    for (int o = kWarps / 2; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const float vmin = __shfl_sync(0xffffffffu, lo, 0), vmax = __shfl_sync(0xffffffffu, hi, 0);
    if (vmin == vmax) { *vtie = vmin == 0.0f ? 0.0f : vmin; return 3; }
    if (!(vmax - vmin < kInf)) return 2;
    const float scale = (float)nb / (vmax - vmin);
    int32_t rb[kRegKeys];
#pragma unroll
    for (int i = 0; i < kRegQuads; ++i) {
        const int32_t e0 = 4 * (i * kThreads + tid);
#pragma unroll
        for (int j = 0; j < 4; ++j) rb[4 * i + j] = nb;     // nb: no key (past the row's end)
        if (i < live) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (e0 + j < n) {
                    rb[4 * i + j] = bucket_of(v[4 * i + j], vmin, scale, nb);
                    if (idx_ok(rb[4 * i + j], nb, sm.dbg)) atomicAdd(&hist[rb[4 * i + j]], 1);
                }
            }
        }
    }
    __syncthreads();
    switch (nb / kThreads) {
        case 1: scan_buckets<1>(hist, m, sm); break;
        case 2: scan_buckets<2>(hist, m, sm); break;
        case 4: scan_buckets<4>(hist, m, sm); break;
        case 8: scan_buckets<8>(hist, m, sm); break;
        default: scan_buckets<16>(hist, m, sm); break;
    }
    __syncthreads();
    if (sm.s_maxbin > kBinCap) return 2;
    const int32_t cutb = sm.s_cut;
#pragma unroll
    for (int i = 0; i < kRegQuads; ++i) {
        if (i < live) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int32_t k = 4 * i + j;
                const int32_t e = 4 * (i * kThreads + tid) + j;
                if (rb[k] <= cutb && idx_ok(rb[k], nb, sm.dbg)) {   // rb == nb past the end
                    const int32_t dst = atomicAdd(&hist[rb[k]], 1);
                    if (idx_ok(dst, m + kBinCap, sm.dbg)) {
                        buf[dst] = ((uint64_t)score_key(v[k]) << 32) | (uint32_t)~(uint32_t)e;
                        bufb[dst] = (uint16_t)rb[k];
                    }
                }
            }
        }
    }
    __syncthreads();
    // rank within the bucket (two composites per step); the top m land in the stage at their
    // output slots, which the caller writes out in slot order
    int32_t filled = hist[cutb];
    if (!in_bounds(filled >= 0 && filled <= m + kBinCap, sm.dbg)) filled = 0;
    for (int32_t p = tid; p < filled; p += kThreads) {
        const uint64_t x = buf[p];
        const int32_t b = bufb[p];
        if (!idx_ok(b, nb, sm.dbg)) continue;
        const int32_t beg = b == 0 ? 0 : hist[b - 1];
        const int32_t end = hist[b];
        if (!in_bounds(beg >= 0 && beg <= end && end <= filled, sm.dbg)) continue;
        int32_t rank = 0;
        int32_t a = beg;
        for (; a + 1 < end; a += 2) rank += (buf[a] > x ? 1 : 0) + (buf[a + 1] > x ? 1 : 0);
        if (a < end) rank += buf[a] > x ? 1 : 0;
        const int32_t slot = beg + rank;
        if (slot < m) stage[slot] = x;
    }
    return 1;
}

// Writes a row's output slots [0, topk): slots below m from the staged composites, the rest
// padding (-1 / -inf), one slot per thread and step (four slots per thread with 16-byte stores
// measured slower).
__device__ __forceinline__ void emit_stage(const uint64_t *stage, int32_t m, int32_t topk,
                                           int32_t off, int32_t *oi, float *ov) {
    const float kNegInf = -__int_as_float(0x7f800000);
    for (int32_t s = threadIdx.x; s < topk; s += kThreads) {
        int32_t id = -1;
        float val = kNegInf;
        if (s < m) {
            const uint64_t x = stage[s];
            id = (int32_t)~(uint32_t)x + off;
            val = key_score((uint32_t)(x >> 32));
        }
        oi[s] = id;
        if (ov) ov[s] = val;
    }
}

// Linear-bucket sort of candidates held in shared memory as (score key << 32 | ~index)
// composites; writes outputs [0, m). Buckets 0..cut are scattered to gbuf/gbufb (shared memory,
// topk + kBinCap entries). Returns 1 when done, 2 when the caller must take the exact path
// (nothing has been written then).
__device__ int cand_bucket_topk(const uint64_t *cand, int32_t n_c, int32_t m, int32_t *hist,
                                uint64_t *gbuf, uint16_t *gbufb, int32_t off, int32_t *oi,
                                float *ov, Smem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float kInf = __int_as_float(0x7f800000);
    float lo = kInf, hi = -kInf;
    for (int32_t p = tid; p < n_c; p += kThreads) {
        const float v = key_score((uint32_t)(cand[p] >> 32));
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) { sm.red_min[warp] = lo; sm.red_max[warp] = hi; }
    int32_t nb = kThreads;
    while (nb < n_c && nb < kNbMax) nb <<= 1;
    for (int i = tid; i < nb / 4; i += kThreads) reinterpret_cast<int4 *>(hist)[i] = make_int4(0, 0, 0, 0);
    if (tid == 0) { sm.s_cut = nb - 1; sm.s_maxbin = 0; }
    __syncthreads();
    if (warp == 0) {
        lo = lane < kWarps ? sm.red_min[lane] : kInf;
        hi = lane < kWarps ? sm.red_max[lane] : -kInf;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (lane == 0) { sm.s_vmin = lo; sm.s_vmax = hi; }
    }
    __syncthreads();
    const float vmin = sm.s_vmin, vmax = sm.s_vmax;
    if (!(vmax - vmin > 0.0f) || !(vmax - vmin < kInf)) return 2;
    const float scale = (float)nb / (vmax - vmin);
    for (int32_t p = tid; p < n_c; p += kThreads) {
        const int32_t rb = bucket_of(key_score((uint32_t)(cand[p] >> 32)), vmin, scale, nb);
        if (idx_ok(rb, nb, sm.dbg)) atomicAdd(&hist[rb], 1);
    }
    __syncthreads();
    switch (nb / kThreads) {
        case 1: scan_buckets<1>(hist, m, sm); break;
        case 2: scan_buckets<2>(hist, m, sm); break;
        case 4: scan_buckets<4>(hist, m, sm); break;
        case 8: scan_buckets<8>(hist, m, sm); break;
        default: scan_buckets<16>(hist, m, sm); break;
    }
    __syncthreads();
    if (sm.s_maxbin > kBinCap) return 2;
    const int32_t cutb = sm.s_cut;
    for (int32_t p = tid; p < n_c; p += kThreads) {
        const uint64_t x = cand[p];
        const int32_t rb = bucket_of(key_score((uint32_t)(x >> 32)), vmin, scale, nb);
        if (rb <= cutb && idx_ok(rb, nb, sm.dbg)) {
            const int32_t dst = atomicAdd(&hist[rb], 1);
            if (idx_ok(dst, m + kBinCap, sm.dbg)) {
                gbuf[dst] = x;
                gbufb[dst] = (uint16_t)rb;
            }
        }
    }
    __syncthreads();
    int32_t filled = hist[cutb];
    if (!in_bounds(filled >= 0 && filled <= m + kBinCap, sm.dbg)) filled = 0;
    for (int32_t p = tid; p < filled; p += kThreads) {
        const uint64_t x = gbuf[p];
        const int32_t b = gbufb[p];
        if (!idx_ok(b, nb, sm.dbg)) continue;
        const int32_t beg = b == 0 ? 0 : hist[b - 1];
        const int32_t end = hist[b];
        if (!in_bounds(beg >= 0 && beg <= end && end <= filled, sm.dbg)) continue;
        int32_t rank = 0;
        for (int32_t a = beg; a < end; ++a) rank += gbuf[a] > x ? 1 : 0;
        const int32_t slot = beg + rank;
        if (slot < m) {
            oi[slot] = (int32_t)~(uint32_t)x + off;
            if (ov) ov[slot] = key_score((uint32_t)(x >> 32));
        }
    }
    return 1;
}

// Long-row path (n > kRegKeys * kThreads). When the row fits the candidate area every key is a
// candidate. Otherwise pass 1 streams the row (float4 loads, several in flight) into a
// histogram of the top 12 bits of the score key (bin 0 = highest); the bin holding rank m-1
// bounds the selection: every key in a higher bin is selected and the needed rest lies in that
// bin. Pass 2 streams the row again and gathers the keys of those bins into shared memory (one
// atomic per warp and iteration). cand_bucket_topk then orders the candidates. Returns 1 when
// done, 2 when the caller must take the exact path.
__device__ int long_row_topk(const float *src, int32_t n, int32_t m, int32_t *hist,
                             uint64_t *cand, int32_t cand_cap, uint64_t *sbuf, uint16_t *sbufb,
                             int32_t off, int32_t *oi, float *ov, Smem &sm) {
    const int tid = threadIdx.x, lane = tid & 31;
    constexpr int kDigitBins = 4096;
    constexpr int kUnroll = 4;
    const float4 *src4 = reinterpret_cast<const float4 *>(src);
    const int32_t n4 = n >> 2;
    if (tid == 0) { sm.s_cut = kDigitBins - 1; sm.s_maxbin = 0; sm.s_append = 0; }
    int32_t cut = kDigitBins;              // every digit bin is taken
    int32_t n_c = n;
    if (n > cand_cap) {
        for (int i = tid; i < kDigitBins / 4; i += kThreads)
            reinterpret_cast<int4 *>(hist)[i] = make_int4(0, 0, 0, 0);
        __syncthreads();
        for (int32_t b4 = tid; b4 < n4; b4 += kUnroll * kThreads) {
            float4 x[kUnroll];
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int32_t i4 = b4 + k * kThreads;
                if (i4 < n4) x[k] = __ldcg(src4 + i4);
            }
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                if (b4 + k * kThreads < n4) {
                    atomicAdd(&hist[(kDigitBins - 1) - (int32_t)(score_key(x[k].x) >> 20)], 1);
                    atomicAdd(&hist[(kDigitBins - 1) - (int32_t)(score_key(x[k].y) >> 20)], 1);
                    atomicAdd(&hist[(kDigitBins - 1) - (int32_t)(score_key(x[k].z) >> 20)], 1);
                    atomicAdd(&hist[(kDigitBins - 1) - (int32_t)(score_key(x[k].w) >> 20)], 1);
                }
            }
        }
        for (int32_t e = 4 * n4 + tid; e < n; e += kThreads)
            atomicAdd(&hist[(kDigitBins - 1) - (int32_t)(score_key(__ldcg(src + e)) >> 20)], 1);
        __syncthreads();
        scan_buckets<kDigitBins / kThreads>(hist, m, sm);
        __syncthreads();
        cut = sm.s_cut;
        n_c = cut + 1 < kDigitBins ? hist[cut + 1] : n;
        if (n_c > cand_cap) return 2;
    } else {
        __syncthreads();
    }
    if (!in_bounds(n_c <= cand_cap, sm.dbg)) return 2;
    // pass 2: keys of bins 0..cut, 16 per thread per iteration: each thread packs its take flags
    // into a mask, a warp scan of the counts gives every thread its write position, and one
    // atomic per warp claims the warp's space
    auto takes = [&](float v) -> bool {
        return (int32_t)((kDigitBins - 1) - (int32_t)(score_key(v) >> 20)) <= cut;
    };
    for (int32_t c0 = 0; c0 < n4; c0 += kUnroll * kThreads) {
        float4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int32_t i4 = c0 + k * kThreads + tid;
            x[k] = i4 < n4 ? __ldcg(src4 + i4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t mask = 0;
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            if (c0 + k * kThreads + tid < n4) {
                mask |= (takes(x[k].x) ? 1u : 0u) << (4 * k + 0);
                mask |= (takes(x[k].y) ? 1u : 0u) << (4 * k + 1);
                mask |= (takes(x[k].z) ? 1u : 0u) << (4 * k + 2);
                mask |= (takes(x[k].w) ? 1u : 0u) << (4 * k + 3);
            }
        }
        const int32_t cnt = __popc(mask);
        int32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const int32_t total = __shfl_sync(0xffffffffu, incl, 31);
        if (total == 0) continue;
        int32_t base = 0;
        if (lane == 31) base = atomicAdd(&sm.s_append, total);
        int32_t pos = __shfl_sync(0xffffffffu, base, 31) + incl - cnt;
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int32_t i4 = c0 + k * kThreads + tid;
            const float vals[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (mask & (1u << (4 * k + c))) {
                    if (pos < n_c)
                        cand[pos] = ((uint64_t)score_key(vals[c]) << 32) | (uint32_t)~(uint32_t)(4 * i4 + c);
                    ++pos;
                }
            }
        }
    }
    {
        const int32_t e = 4 * n4 + tid;         // the last n % 4 keys
        const float v = e < n ? __ldcg(src + e) : 0.0f;
        const bool take = e < n && takes(v);
        const uint32_t bl = __ballot_sync(0xffffffffu, take);
        if (bl) {
            int32_t base = 0;
            if (lane == 0) base = atomicAdd(&sm.s_append, __popc(bl));
            base = __shfl_sync(0xffffffffu, base, 0);
            const int32_t pos = base + __popc(bl & lanemask_lt());
            if (take && pos < n_c) cand[pos] = ((uint64_t)score_key(v) << 32) | (uint32_t)~(uint32_t)e;
        }
    }
    __syncthreads();
    return cand_bucket_topk(cand, n_c, m, hist, sbuf, sbufb, off, oi, ov, sm);
}

// Selection of one row (or one key piece of a row): keys [0, n) of the fp32 row `src`, output
// indices shifted by `off`, topk slots written to oi / ov (ov may be null).
template <bool kLong>
__device__ __forceinline__ void select_body(const Params &sp, int32_t n, int32_t off,
                                            const float *src, int32_t *oi, float *ov,
                                            unsigned char *dsm, Smem &sm) {
    const Problem &p = sp.p;
    const int tid = threadIdx.x;
    const int32_t topk = p.topk;
    // work area shared by the two paths, then the row cache
    int32_t *hist = reinterpret_cast<int32_t *>(dsm);                        // bucket path
    uint64_t *buf = reinterpret_cast<uint64_t *>(hist + kBucketsMax);
    uint16_t *bufb = reinterpret_cast<uint16_t *>(buf + topk + kBinCap);
    uint64_t *stage = reinterpret_cast<uint64_t *>(                        // register path output
        dsm + kBucketsMax * 4 + align_up((size_t)(topk + kBinCap) * 10, 16));
    uint32_t *keyA = reinterpret_cast<uint32_t *>(dsm);                      // exact path
    uint32_t *keyB = keyA + topk;
    int32_t *idxA = reinterpret_cast<int32_t *>(keyB + topk);
    int32_t *idxB = idxA + topk;
    int32_t *cnt = idxB + topk;                                             // kWarps * kDigits
    uint64_t *cand = reinterpret_cast<uint64_t *>(hist + kBucketsMax);       // long-row path
    const uint32_t *rowc = nullptr;                                         // exact path reads global

    const int32_t m = min(n, topk);
    const float kNegInf = -__int_as_float(0x7f800000);

    // 0: all padding, 1: bucket path (outputs written), 2: exact path (A or B buffers),
    // 3: all keys tie
    int mode = 0;
    bool inB = false;
    float vtie = 0.0f;
    int32_t written = 0;
    if (m > 0 && n <= kRegKeys * kThreads) {
        mode = reg_bucket_topk(src, n, m, hist, buf, bufb, stage, sm, &vtie);
        if (mode == 1) {
            __syncthreads();
            emit_stage(stage, m, topk, off, oi, ov);
            written = topk;
        }
        if (mode == 2) {
            uint32_t prefix = 0u, mask = 0u;
            int32_t need = m;
            if (m < n) radix_select<false>(rowc, src, n, m, sm, prefix, mask, need);
            gather<false>(rowc, src, n, m, prefix, mask, need, keyA, idxA, sm);
            __syncthreads();
            inB = sort_desc(m, keyA, idxA, keyB, idxB, cnt, sm);
        }
    } else if (kLong && m > 0) {
        uint64_t *sbuf = cand + sp.cand_cap;
        uint16_t *sbufb = reinterpret_cast<uint16_t *>(sbuf + topk + kBinCap);
        mode = long_row_topk(src, n, m, hist, cand, sp.cand_cap, sbuf, sbufb, off, oi, ov, sm);
        if (mode == 1) written = m;
        if (mode == 2) {
            uint32_t prefix = 0u, mask = 0u;
            int32_t need = m;
            if (m < n) radix_select<false>(rowc, src, n, m, sm, prefix, mask, need);
            gather<false>(rowc, src, n, m, prefix, mask, need, keyA, idxA, sm);
            __syncthreads();
            inB = sort_desc(m, keyA, idxA, keyB, idxB, cnt, sm);
        }
    }
    if (mode == 2 && tid == 0) atomicAdd(&sp.ws->exact_rows, 1);
    const uint32_t *kf = inB ? keyB : keyA;
    const int32_t *jf = inB ? idxB : idxA;
    // the bucket paths have written slots [0, written) already
    for (int32_t s = written + tid; s < topk; s += kThreads) {
        int32_t id = -1;
        float v = kNegInf;
        if (s < m) {
            if (mode == 2) {
                id = jf[s] + off;
                v = key_score(kf[s]);
            } else {
                id = s + off;
                v = vtie;
            }
        }
        oi[s] = id;
        if (ov) ov[s] = v;
    }
}

// Window and output offset of query row r: *n keys, *off added to the indices. Checks the
// schedule's signature (block 0 reports it) and, without a schedule kernel, the row's offset.
__device__ __forceinline__ void row_window(const Params &sp, int32_t r, int32_t *n, int32_t *off) {
    const Problem &p = sp.p;
    const int tid = threadIdx.x;
    bool meta_ok = true;
    if (sp.view.meta) {
        const MetaHeader *hdr = reinterpret_cast<const MetaHeader *>(sp.view.meta);
        meta_ok = hdr->magic == kMetaMagic && hdr->signature == sp.signature;
        if (blockIdx.x == 0 && tid == 0)
            set_status(&sp.ws->status, meta_ok ? hdr->status : kDevErrMetadata);
    }
    int32_t pos = 0;
    int32_t b = meta_ok ? row_batch(p, r, &pos) : -1;
    *n = 0;
    *off = 0;
    if (b >= 0) {
        const BatchInfo bi = sp.view.batch(p, b);
        *n = window_hi(p.mask_mode, pos, bi.L1u, bi.L2, p.cmp_ratio, bi.pad[2]);

        if (p.output_idx_offset) {
            *off = p.output_idx_offset[b];
            // the schedule kernel validates offsets; without it each row checks its own
            if (!sp.view.meta && tid == 0 &&
                (*off < 0 || (int64_t)*off + (bi.L2 > 0 ? bi.L2 - 1 : 0) > (int64_t)INT32_MAX))
                set_status(&sp.ws->status, LI_DEVERR_OFFSET);
        }
    }
}

// kLong: the problem may have rows longer than kRegKeys * kThreads keys (long-row path compiled
// in; two CTAs per SM). Otherwise only the register path and the exact fallback exist.
template <bool kLong>
__global__ void __launch_bounds__(kThreads, kLong ? (kThreads >= 1024 ? 1 : 2) : 4) select_kernel(Params sp) {
    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ Smem sm;
    // blocks start in index order; later rows of a causal window are the longer ones, so the
    // rows are taken last to first (longest first)
    const int32_t r = (int32_t)(gridDim.x - 1 - blockIdx.x);
    if constexpr (kDebugBounds) {
        if (threadIdx.x == 0) sm.dbg = &sp.ws->status;
        __syncthreads();
    }
    int32_t n, off;
    row_window(sp, r, &n, &off);
    const int32_t topk = sp.p.topk;
    select_body<kLong>(sp, n, off, sp.scores + (int64_t)r * sp.ld, sp.out_idx + (int64_t)r * topk,
                       sp.out_val ? sp.out_val + (int64_t)r * topk : nullptr, dsm, sm);
}

// Few very long rows: each row's keys are cut into `pieces` consecutive pieces of piece_len keys
// (a multiple of 128, so every piece starts 16-byte aligned), one CTA per (row, piece). Piece
// c of row r selects among keys [c*piece_len, min(n, (c+1)*piece_len)) with their row indices
// and writes a full top-k list (sorted, padded) to list c of the partial buffers
// [pieces][rows][topk]; the split merge turns the lists into the row's output.
template <bool kLong>
__global__ void __launch_bounds__(kThreads, kLong ? (kThreads >= 1024 ? 1 : 2) : 4)
select_piece_kernel(Params sp, PieceParams pp) {
    extern __shared__ __align__(16) unsigned char dsm[];
    __shared__ Smem sm;
    const int32_t rows = (int32_t)(gridDim.x / pp.pieces);
    const int32_t r = rows - 1 - (int32_t)(blockIdx.x / pp.pieces);
    const int32_t c = (int32_t)(blockIdx.x % pp.pieces);
    if constexpr (kDebugBounds) {
        if (threadIdx.x == 0) sm.dbg = &sp.ws->status;
        __syncthreads();
    }
    int32_t n, off;
    row_window(sp, r, &n, &off);
    const int64_t start = (int64_t)c * pp.piece_len;
    const int32_t len = n > start ? (int32_t)min((int64_t)pp.piece_len, (int64_t)n - start) : 0;
    const int64_t slot = ((int64_t)c * rows + r) * sp.p.topk;
    select_body<kLong>(sp, len, off + (int32_t)start, sp.scores + (int64_t)r * sp.ld + start,
                       pp.idx + slot, pp.val + slot, dsm, sm);
}

// Bytes of the dynamic shared memory work area: the largest of the short-row bucket path
// (histogram + scattered composites + their buckets + the output stage), the long-row path
// (histogram + candidates + scattered composites + their buckets) and the exact path (two
// key/index buffers + digit counters).
static size_t select_work_bytes(int topk, bool long_rows, int32_t *cand_cap) {
    const size_t scatter = (size_t)(topk + kBinCap) * 10;
    const size_t staged = (size_t)(topk < kRegKeys * kThreads ? topk : kRegKeys * kThreads) * 8;
    const size_t shortp = (size_t)kBucketsMax * 4 + align_up(scatter, 16) + staged;
    const size_t exact = (size_t)4 * topk * 4 + (size_t)kWarps * kDigits * 4;
    size_t work = shortp > exact ? shortp : exact;
    *cand_cap = 0;
    if (long_rows) {
        // candidates: the m selected plus the rest of the threshold digit bin
        constexpr size_t kBudget = 200 * 1024;
        int64_t cap = 2LL * topk + 4096;
        const int64_t fit = ((int64_t)kBudget - kBucketsMax * 4 - (int64_t)scatter) / 8;
        if (cap > fit) cap = fit;
        cap = cap / 32 * 32;
        const size_t longp = (size_t)kBucketsMax * 4 + (size_t)cap * 8 + scatter;
        if (longp > work) work = longp;
        *cand_cap = (int32_t)cap;
    }
    return align_up(work, 16);
}

