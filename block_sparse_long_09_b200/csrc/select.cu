// select.cu -- QSA top-k micro-block selection.
//
// Budget sentence of "On the Design of Qwen3.8 Next Architecture" (reading
// notes, section 6): per query, the own (trailing, possibly incomplete) causal
// block b_t is always kept and the remaining k - 1 slots go to the best complete
// blocks 0 .. b_t - 1.  Ties go to the lower block index; the output lists the
// chosen blocks in ascending order, padded with -1.
//
// One CTA per query row, about 41 KB of shared memory: 128 threads when there
// are many rows (prefill), so several rows are in flight on every SM and their
// memory latency overlaps; 512 threads when rows are few (decode).  The fp32
// scores become order-preserving 32-bit keys (sign-flip trick, -0.0 folded
// into +0.0).
//  * Fast path (rows of up to 65536 candidates): a strided sample of 1024 keys
//    yields a conservative lower bound on the threshold (its rank in the
//    sample is 4 sigma above the expected one); one pass over the row (32 keys
//    in flight per thread, a float compare per key and a warp vote per four)
//    lists every key at or above the bound with warp-aggregated appends; the exact (k-1)-th key is then found on that
//    short list by an MSD radix select with 8-bit digits.  Each score is read
//    from global memory once.
//  * General path (the bound missed, the list overflowed, or a longer row):
//    the same radix select over every key, read from global memory per digit.
// Winners land in two bitmaps -- "above the threshold" and "equal to it" -- and
// only when the threshold value is shared by more keys than slots left does a
// scan of the "equal" bitmap pick the lowest indices; one block scan of the
// bitmap popcounts gives every winner its output position, so the list comes
// out ascending without a sort.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kMaxSelWarps = 16;
constexpr int kBins = 256;                   // 8-bit digits
constexpr int kSegWords = 2048;              // bitmap segment: 65536 candidates
constexpr int kSegElems = kSegWords * 32;
constexpr int kCandCap = 3072;               // fast-path list
constexpr int kSampleMax = 1024;             // strided sample that bounds the threshold
constexpr int kSelSmem = (kBins + 2 * kSegWords + 2 * kCandCap) * 4;  // 41 KB

__device__ __forceinline__ uint32_t order_key(float x)
{
    uint32_t b = __float_as_uint(x);
    if ((b << 1) == 0u) b = 0u;  // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// inverse of order_key (for keys of non-NaN floats): x >= key_value(k) <=> order_key(x) >= k
__device__ __forceinline__ float key_value(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct SelScratch {
    int warp_tot[kMaxSelWarps];
    int digit, above;
    int cand_n;
};

// block-wide exclusive scan of one int per thread; every thread gets the total
template <int kSelThreads>
__device__ __forceinline__ int block_exclusive_scan(int v, SelScratch *sc, int *total)
{
    constexpr int kSelWarps = kSelThreads / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) sc->warp_tot[wid] = incl;
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
        const int c = sc->warp_tot[w];
        before += (w < wid) ? c : 0;
        tot += c;
    }
    __syncthreads();
    *total = tot;
    return before + incl - v;
}

// hist[0 .. 256) counts the keys still in play by digit: find the digit whose bin
// holds the need-th largest key.  *above = keys in higher bins.
template <int kSelThreads>
__device__ __forceinline__ int find_digit(const uint32_t *hist, int need, SelScratch *sc, int *above_out)
{
    const int tid = threadIdx.x;
    constexpr int per = kBins >= kSelThreads ? kBins / kSelThreads : 1;  // digits per thread, highest first
    const int top = kBins - tid * per;                                  // owns digits [top - per, top)
    const bool owns = top > 0;
    int mine = 0;
#pragma unroll
    for (int q = 1; q <= per; ++q) mine += owns ? (int)hist[top - q] : 0;
    int tot;
    int above = block_exclusive_scan<kSelThreads>(mine, sc, &tot);
#pragma unroll
    for (int q = 1; q <= per; ++q) {
        if (!owns) break;
        const int h = (int)hist[top - q];
        if (above < need && above + h >= need) {
            sc->digit = top - q;
            sc->above = above;
        }
        above += h;
    }
    __syncthreads();
    const int d = sc->digit;
    *above_out = sc->above;
    __syncthreads();
    return d;
}

// MSD radix select over keys get(0 .. count): locate the need-th largest key.
// Returns the resolved digits as prefix/mask; *need_left = keys equal to the
// prefix still needed, *in_bin = keys equal to the prefix.
template <int kSelThreads, typename Get>
__device__ __forceinline__ void radix_select(Get get, int count, int need, uint32_t *hist, SelScratch *sc,
                                             uint32_t *prefix_out, uint32_t *mask_out, int *need_left,
                                             int *in_bin_out)
{
    const int tid = threadIdx.x;
    uint32_t prefix = 0u, mask = 0u;
    int in_bin = count;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = tid; b < kBins; b += kSelThreads) hist[b] = 0u;
        __syncthreads();
        for (int i = tid; i < count; i += kSelThreads) {
            const uint32_t u = get(i);
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 0xFFu], 1u);
        }
        __syncthreads();
        int ab;
        const int d = find_digit<kSelThreads>(hist, need, sc, &ab);
        need -= ab;
        prefix |= (uint32_t)d << shift;
        mask |= 0xFFu << shift;
        in_bin = (int)hist[d];
        __syncthreads();
        if (need == in_bin) break;  // the whole bin is taken: no finer digit matters
    }
    *prefix_out = prefix;
    *mask_out = mask;
    *need_left = need;
    *in_bin_out = in_bin;
}

// Ordered emission of one bitmap segment: winners are gtw bits plus, when
// `partial`, the lowest-index eqw bits while the running equal-rank stays below
// `need`; otherwise all eqw bits.  Writes out[pos] = seg0 + bit index.
template <int kSelThreads>
__device__ __forceinline__ void emit_segment(const uint32_t *gtw, const uint32_t *eqw, int words, int seg0,
                                             bool partial, int need, int need_total, int *out_base,
                                             int *eq_base, int32_t *out, SelScratch *sc)
{
    constexpr int kWordsPerThread = kSegWords / kSelThreads;
    const int tid = threadIdx.x;
    uint32_t wsel[kWordsPerThread];
    const int w0 = tid * kWordsPerThread;
    if (partial) {
        int ecnt = 0;
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) ecnt += (w0 + q < words) ? __popc(eqw[w0 + q]) : 0;
        int etot;
        int epos = *eq_base + block_exclusive_scan<kSelThreads>(ecnt, sc, &etot);
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) {
            uint32_t e = (w0 + q < words) ? eqw[w0 + q] : 0u;
            uint32_t taken = 0u;
            while (e != 0u && epos < need) {  // keep the lowest set bits while rank < need
                const uint32_t lowbit = e & (~e + 1u);
                taken |= lowbit;
                e ^= lowbit;
                ++epos;
            }
            epos += __popc(e);
            wsel[q] = ((w0 + q < words) ? gtw[w0 + q] : 0u) | taken;
        }
        *eq_base += etot;
    } else {
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) wsel[q] = (w0 + q < words) ? (gtw[w0 + q] | eqw[w0 + q]) : 0u;
    }
    int cnt = 0;
#pragma unroll
    for (int q = 0; q < kWordsPerThread; ++q) cnt += __popc(wsel[q]);
    int stot;
    int pos = *out_base + block_exclusive_scan<kSelThreads>(cnt, sc, &stot);
#pragma unroll
    for (int q = 0; q < kWordsPerThread; ++q) {
        uint32_t b = wsel[q];
        while (b != 0u) {
            const int bit = __ffs(b) - 1;
            b &= b - 1u;
            if (pos < need_total) out[pos] = seg0 + (w0 + q) * 32 + bit;
            ++pos;
        }
    }
    *out_base += stot;
}

template <int kSelThreads>
__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ cu_q,
              const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r,
              int32_t *__restrict__ sel)
{
    extern __shared__ uint32_t smem_sel[];
    uint32_t *hist = smem_sel;                     // kBins
    uint32_t *gtw = hist + kBins;                  // kSegWords: key above the threshold
    uint32_t *eqw = gtw + kSegWords;               // kSegWords: key equal to the threshold
    uint32_t *cand_key = eqw + kSegWords;          // kCandCap (the sample first)
    uint32_t *cand_idx = cand_key + kCandCap;      // kCandCap
    __shared__ SelScratch sc;
    constexpr int kSelWarps = kSelThreads / 32;

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t i = row_begin + blockIdx.x;
    int s;
    int64_t t;
    if (cu_q != nullptr) {
        s = find_seq(cu_q, batch, i);
        const int64_t Lq = (int64_t)cu_q[s + 1] - cu_q[s];
        const int64_t Lk = (int64_t)cu_k[s + 1] - cu_k[s];
        t = (Lk - Lq) + (i - cu_q[s]);
    } else {
        s = (int)i;
        t = (int64_t)cu_k[s + 1] - cu_k[s] - 1;
    }
    if (t < 0) {
        if (tid == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        return;
    }
    const int64_t bt = t / r;
    if (bt > ld || bt > 0x7FFFFFFF) {  // scores row too short for this query
        if (tid == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        return;
    }
    const float *srow = scores + (int64_t)blockIdx.x * ld;
    int32_t *out = sel + i * k;
    const int need_total = k - 1;

    if (bt <= need_total) {  // every candidate fits: 0 .. b_t, then padding
        for (int j = tid; j < k; j += kSelThreads) out[j] = (j <= bt) ? j : -1;
        return;
    }
    const int n = (int)bt;
    int out_base = 0, eq_base = 0;

    // ============================ fast path ============================
    bool done = false;
    if (n <= kSegElems) {
        const int ns = n < kSampleMax ? n : kSampleMax;
        for (int w = tid; w < kSegWords; w += kSelThreads) {
            gtw[w] = 0u;
            eqw[w] = 0u;
        }
        const int stride = n / ns;
        for (int q = tid; q < ns; q += kSelThreads) cand_key[q] = order_key(__ldg(srow + q * stride));
        if (tid == 0) sc.cand_n = 0;
        __syncthreads();
        // bound: the r_lo-th largest sample key, r_lo = mean + 4 sigma + 8 ranks.  When
        // the radix select stops on a bin taken whole, the prefix (the bin's smallest
        // possible key) is a bound as well.
        const float mu = (float)need_total * (float)ns / (float)n;
        int r_lo = (int)ceilf(mu + 4.f * sqrtf(mu) + 8.f);
        if (r_lo > ns) r_lo = ns;
        uint32_t lo_key;
        {
            uint32_t mk;
            int nl, ib;
            radix_select<kSelThreads>([&](int q) { return cand_key[q]; }, ns, r_lo, hist, &sc, &lo_key, &mk, &nl, &ib);
        }
        __syncthreads();
        // one pass over the row: list every key >= lo_key.  Most keys are below the
        // bound, so the test is a float compare (lo_val is the bound's value; -0.0
        // compares equal to +0.0, like the keys) with one vote per 4 keys, and only a
        // warp that holds a candidate pays for the ballots and appends.
        const float lo_val = key_value(lo_key);
        auto append = [&](float x, int j, bool c) {
            const uint32_t cb = __ballot_sync(0xffffffffu, c);
            if (cb == 0u) return;
            int base = 0;
            if (lane == 0) base = atomicAdd(&sc.cand_n, __popc(cb));
            base = __shfl_sync(0xffffffffu, base, 0);
            const int p = base + __popc(cb & ((1u << lane) - 1u));
            if (c && p < kCandCap) {
                cand_key[p] = order_key(x);
                cand_idx[p] = (uint32_t)j;
            }
        };
        if ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {
            const float4 *s4 = reinterpret_cast<const float4 *>(srow);
            const int n4 = (n + 3) >> 2;
            const int n4full = n >> 2;
            constexpr float kNeg = -INFINITY;
            for (int j0 = tid; j0 - tid < n4; j0 += 8 * kSelThreads) {  // uniform trip count
                float4 v[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {  // 32 keys in flight per thread
                    const int j4 = j0 + q * kSelThreads;
                    v[q] = j4 < n4full ? __ldg(s4 + j4) : make_float4(kNeg, kNeg, kNeg, kNeg);
                    if (j4 == n4full && j4 < n4) {  // ragged tail, element by element
                        const int e = j4 * 4;
                        v[q].x = e < n ? __ldg(srow + e) : kNeg;
                        v[q].y = e + 1 < n ? __ldg(srow + e + 1) : kNeg;
                        v[q].z = e + 2 < n ? __ldg(srow + e + 2) : kNeg;
                    }
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const bool cx = v[q].x >= lo_val, cy = v[q].y >= lo_val;
                    const bool cz = v[q].z >= lo_val, cw = v[q].w >= lo_val;
                    if (!__any_sync(0xffffffffu, cx || cy || cz || cw)) continue;
                    const int e = (j0 + q * kSelThreads) * 4;
                    append(v[q].x, e, cx);
                    append(v[q].y, e + 1, cy);
                    append(v[q].z, e + 2, cz);
                    append(v[q].w, e + 3, cw);
                }
            }
        } else {
            for (int j0 = tid; j0 - tid < n; j0 += 4 * kSelThreads) {  // uniform trip count
                float v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int j = j0 + q * kSelThreads;
                    v[q] = j < n ? __ldg(srow + j) : -INFINITY;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const bool c = v[q] >= lo_val;
                    if (!__any_sync(0xffffffffu, c)) continue;
                    append(v[q], j0 + q * kSelThreads, c);
                }
            }
        }
        __syncthreads();
        const int nc = sc.cand_n;
        if (nc >= need_total && nc <= kCandCap) {
            // exact threshold among the listed keys (every key above it is listed)
            uint32_t prefix, mask;
            int need, in_bin;
            radix_select<kSelThreads>([&](int c) { return cand_key[c]; }, nc, need_total, hist, &sc, &prefix, &mask, &need,
                         &in_bin);
            const bool partial = need < in_bin;
            for (int c = tid; c < nc; c += kSelThreads) {
                const uint32_t u = cand_key[c] & mask;
                const uint32_t j = cand_idx[c];
                if (u > prefix) atomicOr(&gtw[j >> 5], 1u << (j & 31));
                else if (u == prefix) atomicOr(&eqw[j >> 5], 1u << (j & 31));
            }
            __syncthreads();
            emit_segment<kSelThreads>(gtw, eqw, (n + 31) >> 5, 0, partial, need, need_total, &out_base, &eq_base, out, &sc);
            done = true;
        }
        __syncthreads();
    }

    // ============================ general path ============================
    if (!done) {
        uint32_t prefix, mask;
        int need, in_bin;
        radix_select<kSelThreads>([&](int j) { return order_key(__ldg(srow + j)); }, n, need_total, hist, &sc, &prefix, &mask,
                     &need, &in_bin);
        const bool partial = need < in_bin;
        for (int seg0 = 0; seg0 < n; seg0 += kSegElems) {
            const int seg_n = n - seg0 < kSegElems ? n - seg0 : kSegElems;
            const int words = (seg_n + 31) >> 5;
            for (int w = wid; w < words; w += kSelWarps) {
                const int j = seg0 + w * 32 + lane;
                const bool in = j < n;
                const uint32_t u = in ? (order_key(__ldg(srow + j)) & mask) : 0u;
                const uint32_t g = __ballot_sync(0xffffffffu, in && u > prefix);
                const uint32_t e = __ballot_sync(0xffffffffu, in && u == prefix);
                if (lane == 0) {
                    gtw[w] = g;
                    eqw[w] = e;
                }
            }
            __syncthreads();
            emit_segment<kSelThreads>(gtw, eqw, words, seg0, partial, need, need_total, &out_base, &eq_base, out, &sc);
            __syncthreads();
        }
    }
    if (tid == 0) {
        if (out_base != need_total) set_device_status(QSA_ERR_DEVICE_CHECK);
        out[need_total] = (int32_t)bt;
    }
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0) return cudaSuccess;
    // many rows (prefill): small CTAs, several rows per SM; few rows (decode): wide CTAs
    const bool wide = rows < 4 * num_sms();
    for (int64_t done = 0; done < rows; done += 0x7FFFFFFF) {
        const int64_t chunk = rows - done < 0x7FFFFFFF ? rows - done : 0x7FFFFFFF;
        if (wide)
            select_kernel<512><<<(unsigned)chunk, 512, kSelSmem, stream>>>(
                a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, a.sel);
        else
            select_kernel<128><<<(unsigned)chunk, 128, kSelSmem, stream>>>(
                a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, a.sel);
    }
    return cudaGetLastError();
}

}  // namespace qsa
