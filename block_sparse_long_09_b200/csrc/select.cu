// select.cu -- QSA top-k micro-block selection.
//
// Budget sentence of "On the Design of Qwen3.8 Next Architecture" (reading
// notes, section 6): per query, the own (trailing, possibly incomplete) causal
// block b_t is always kept and the remaining k - 1 slots go to the best complete
// blocks 0 .. b_t - 1.  Ties go to the lower block index; the output lists the
// chosen blocks in ascending order, padded with -1.
//
// One CTA per query row, about 25 KB of shared memory: 128 threads when there
// are many rows (prefill), so eight rows are in flight on every SM and their
// memory latency overlaps; 512 threads when rows are few (decode).  The fp32
// scores become order-preserving 32-bit keys (sign-flip trick, -0.0 folded
// into +0.0).
//  * Fast path (16-byte aligned rows of up to 65536 candidates):
//    - bound: a sample of 1024..2048 keys in runs of 8 spread over the row (a
//      run is one 32-byte sector); two 8-bit digits of a radix select over the
//      sample keys relative to their minimum locate the sample of rank r_lo (4
//      sigma above the expected rank of the threshold), and the smallest sample
//      of that bin is a conservative lower bound;
//    - one pass over the row (32 keys in flight per thread): for every key slot
//      a warp ballot of key >= bound gives each candidate its place in the
//      warp's private list, and the lane that holds it writes score and index
//      there from its registers (nothing is read twice);
//    - an MSD radix select with 8-bit digits over the candidates' keys relative
//      to the bound, started at their highest differing bit, finds the exact
//      (k-1)-th key; the winners' bits are set in a bitmap, and a block scan of
//      its word popcounts gives every winner its output slot, so the list comes
//      out ascending without a sort.
//  * General path (the bound missed, a list overflowed, the threshold value is
//    shared by more keys than slots left, an unaligned or a longer row): a
//    radix select with 11-bit digits over every key, read from global memory
//    per digit, then bitmaps of the keys above and equal to the threshold per
//    65536-key segment; the lowest indices win among equal keys.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kMaxSelWarps = 16;
constexpr int kBins = 2048;                  // 11-bit digits (sample pass, general path)
constexpr int kCandBits = 8;                 // digits of the exact select over the candidates
constexpr int kSegWords = 2048;              // bitmap segment: 65536 candidates
constexpr int kSegElems = kSegWords * 32;
constexpr int kCandCap = 2048;               // candidate lists (and the sample)
constexpr int kSampleMin = 1024;

// shared memory: region A (kSegWords words: histogram, then the winner bitmap)
// and region C (kCandCap (score bits, index) pairs; before them the sample keys,
// after them the bitmap word prefixes; in the general path the "equal" bitmap)
template <int kSelThreads>
constexpr int sel_smem_bytes()
{
    return kSegWords * 4 + kCandCap * 8;
}
static_assert(kBins <= kSegWords, "the histogram lives in region A");
static_assert(kCandCap * 2 >= kSegWords && kCandCap * 2 >= kCandCap, "samples, prefixes and eqw fit region C");

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

// st.shared.v2 of (a, b) at addr when p holds: a predicated store, no branch
__device__ __forceinline__ void st_shared_v2_if(bool p, uint32_t addr, uint32_t a, uint32_t b)
{
    asm volatile(
        "{\n\t.reg .pred q;\n\t"
        "setp.ne.u32 q, %0, 0;\n\t"
        "@q st.shared.v2.u32 [%1], {%2, %3};\n\t}" ::"r"((uint32_t)p),
        "r"(addr), "r"(a), "r"(b)
        : "memory");
}

struct SelScratch {
    int warp_tot[kMaxSelWarps];
    uint32_t warp_val[kMaxSelWarps];
    int warp_cnt[kMaxSelWarps];  // candidates listed per warp
    int digit, above;
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

// block-wide sum (or max) of one value per thread (warp-uniform inputs allowed)
template <int kSelThreads, bool kMax>
__device__ __forceinline__ uint32_t block_reduce(uint32_t v, SelScratch *sc)
{
    constexpr int kSelWarps = kSelThreads / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    v = kMax ? __reduce_max_sync(0xffffffffu, v) : __reduce_add_sync(0xffffffffu, v);
    if (lane == 0) sc->warp_val[wid] = v;
    __syncthreads();
    uint32_t r = 0u;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) r = kMax ? (r > sc->warp_val[w] ? r : sc->warp_val[w]) : r + sc->warp_val[w];
    __syncthreads();
    return r;
}

// block-wide max of two values per thread, in one round
template <int kSelThreads>
__device__ __forceinline__ void block_max2(uint32_t &a, uint32_t &b, SelScratch *sc)
{
    constexpr int kSelWarps = kSelThreads / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    a = __reduce_max_sync(0xffffffffu, a);
    b = __reduce_max_sync(0xffffffffu, b);
    if (lane == 0) {
        sc->warp_val[wid] = a;
        sc->warp_tot[wid] = (int)b;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
        a = a > sc->warp_val[w] ? a : sc->warp_val[w];
        b = b > (uint32_t)sc->warp_tot[w] ? b : (uint32_t)sc->warp_tot[w];
    }
    __syncthreads();
}

// hist[0 .. nb) counts the keys still in play by digit (nb a power of two <=
// 2^kBitsMax): find the digit whose bin holds the need-th largest key (1 <= need
// <= keys in play).  *above = keys in higher bins.
template <int kSelThreads, int kBitsMax>
__device__ __forceinline__ int find_digit(const uint32_t *hist, int nb, int need, SelScratch *sc, int *above_out)
{
    constexpr int kPer = (1 << kBitsMax) >= kSelThreads ? (1 << kBitsMax) / kSelThreads : 1;
    const int tid = threadIdx.x;
    const int per = (nb + kSelThreads - 1) / kSelThreads;
    const int top = nb - tid * per;  // this thread owns bins [top - per, top), highest first
    int mine = 0;
#pragma unroll
    for (int q = 1; q <= kPer; ++q)
        if (q <= per && top - q >= 0) mine += (int)hist[top - q];
    int tot;
    int above = block_exclusive_scan<kSelThreads>(mine, sc, &tot);
#pragma unroll
    for (int q = 1; q <= kPer; ++q) {
        if (q <= per && top - q >= 0) {
            const int h = (int)hist[top - q];
            if (above < need && above + h >= need) {
                sc->digit = top - q;
                sc->above = above;
            }
            above += h;
        }
    }
    __syncthreads();
    const int d = sc->digit;
    *above_out = sc->above;
    __syncthreads();
    return d;
}

// MSD radix select over the keys that visit(f) hands to f (each thread its own
// share), whose bits above `top` are all zero: locate the need-th largest key
// (1 <= need <= count) with kBits-bit digits from bit `top` down, at most
// max_passes digits.  Returns the resolved bits as prefix/mask (the prefix alone
// is a lower bound on the key); *need_left = keys equal to the prefix still
// needed, *in_bin = keys equal to it.
template <int kSelThreads, int kBits, typename Visit>
__device__ __forceinline__ void radix_select(Visit visit, int count, int need, int top, uint32_t *hist,
                                             SelScratch *sc, uint32_t *prefix_out, uint32_t *mask_out,
                                             int *need_left, int *in_bin_out, int max_passes = 32)
{
    const int tid = threadIdx.x;
    uint32_t prefix = 0u;
    uint32_t mask = top >= 31 ? 0u : ~((2u << top) - 1u);
    int in_bin = count;
    int hi = top;
#pragma unroll 1
    while (true) {
        const int lo = hi - (kBits - 1) > 0 ? hi - (kBits - 1) : 0;
        const int nb = 1 << (hi - lo + 1);
        for (int b = tid; b < nb; b += kSelThreads) hist[b] = 0u;
        __syncthreads();
        visit([&](uint32_t u) {
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> lo) & (uint32_t)(nb - 1)], 1u);
        });
        __syncthreads();
        int ab;
        const int d = find_digit<kSelThreads, kBits>(hist, nb, need, sc, &ab);
        need -= ab;
        prefix |= (uint32_t)d << lo;
        mask |= (uint32_t)(nb - 1) << lo;
        in_bin = (int)hist[d];
        __syncthreads();
        if (need == in_bin || lo == 0 || --max_passes == 0) break;  // bin taken whole, or resolved
        hi = lo - 1;
    }
    *prefix_out = prefix;
    *mask_out = mask;
    *need_left = need;
    *in_bin_out = in_bin;
}

// Ordered emission of one bitmap segment: winners are gtw bits plus, when
// `partial`, the lowest-index eqw bits while the running equal-rank stays below
// `need` (otherwise gtw already holds the equal keys).  Writes out[pos] = seg0 +
// bit index.
template <int kSelThreads>
__device__ __forceinline__ void emit_segment(const uint32_t *gtw, const uint32_t *eqw, int words, int seg0,
                                             bool partial, int need, int need_total, int *out_base,
                                             int *eq_base, int32_t *out, SelScratch *sc)
{
    constexpr int kWordsPerThread = kSegWords / kSelThreads;  // at most
    const int tid = threadIdx.x;
    uint32_t wsel[kWordsPerThread];
    const int wpt = (words + kSelThreads - 1) / kSelThreads;  // spread the words over every thread
    const int w0 = tid * wpt;
    const int wend = min(w0 + wpt, words);
    if (partial) {
        int ecnt = 0;
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) ecnt += (w0 + q < wend) ? __popc(eqw[w0 + q]) : 0;
        int etot;
        int epos = *eq_base + block_exclusive_scan<kSelThreads>(ecnt, sc, &etot);
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) {
            uint32_t e = (w0 + q < wend) ? eqw[w0 + q] : 0u;
            uint32_t taken = 0u;
            while (e != 0u && epos < need) {  // keep the lowest set bits while rank < need
                const uint32_t lowbit = e & (~e + 1u);
                taken |= lowbit;
                e ^= lowbit;
                ++epos;
            }
            epos += __popc(e);
            wsel[q] = ((w0 + q < wend) ? gtw[w0 + q] : 0u) | taken;
        }
        *eq_base += etot;
    } else {  // every key equal to the threshold wins: they are in gtw already
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) wsel[q] = (w0 + q < wend) ? gtw[w0 + q] : 0u;
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
__global__ void __launch_bounds__(kSelThreads, kSelThreads == 128 ? 8 : 2)
select_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ cu_q,
              const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r,
              int32_t *__restrict__ sel)
{
    constexpr int kSelWarps = kSelThreads / 32;
    constexpr int kCapW = kCandCap / kSelWarps;         // candidate list of one warp
    extern __shared__ uint32_t smem_sel[];
    uint32_t *regA = smem_sel;                          // kSegWords words
    uint2 *cand = reinterpret_cast<uint2 *>(regA + kSegWords);  // kCandCap (score bits, index)
    uint32_t *regB = reinterpret_cast<uint32_t *>(cand);         // the same bytes, as words
    __shared__ SelScratch sc;

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
    if (n <= kSegElems && (reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {
        // ---- bound from a sample: about 16 expected winners, 1024..2048 keys ----
        int ns = (int)min((int64_t)kCandCap, max((int64_t)kSampleMin, (int64_t)16 * n / need_total));
        uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
        if (n <= kCandCap) {  // short row: the sample is the whole row
            ns = n;
            for (int q = tid; q < ns; q += kSelThreads) {
                const uint32_t u = order_key(__ldg(srow + q));
                regB[q] = u;
                kmin = u < kmin ? u : kmin;
                kmax = u > kmax ? u : kmax;
            }
        } else {  // runs of 8 keys (two float4, one sector) at ns / 8 spread places
            const int runs = ns >> 3;
            ns = runs << 3;
            for (int g = tid; g < runs; g += kSelThreads) {
                const int at = (int)(((int64_t)g * n) / runs) & ~3;  // 16-byte aligned, at + 8 <= n
                const float4 a = __ldg(reinterpret_cast<const float4 *>(srow + at));
                const float4 b = __ldg(reinterpret_cast<const float4 *>(srow + at + 4));
                const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t u = order_key(x[e]);
                    regB[g * 8 + e] = u;
                    kmin = u < kmin ? u : kmin;
                    kmax = u > kmax ? u : kmax;
                }
            }
        }
        kmin = ~kmin;
        block_max2<kSelThreads>(kmin, kmax, &sc);
        kmin = ~kmin;
        // r_lo = mean + 4 sigma + 8 ranks
        const float mu = (float)need_total * (float)ns / (float)n;
        int r_lo = (int)ceilf(mu + 4.f * sqrtf(mu) + 8.f);
        if (r_lo > ns) r_lo = ns;
        uint32_t lo_key;
        {
            const uint32_t sspan = kmax - kmin;
            uint32_t mk;
            int nl, ib;
            radix_select<kSelThreads, 8>(
                [&](auto f) {
                    for (int q = tid; q < ns; q += kSelThreads) f(regB[q] - kmin);
                },
                ns, r_lo, sspan != 0u ? 31 - __clz(sspan) : 0, regA, &sc, &lo_key, &mk, &nl, &ib, 2);
            if (mk != 0xFFFFFFFFu) {
                // stopped on a bin with the sample of rank r_lo in it: its smallest key
                // ranks r_lo or a little below (the bin's floor would be a looser bound)
                uint32_t mn = 0xFFFFFFFFu;
                for (int q = tid; q < ns; q += kSelThreads) {
                    const uint32_t u = regB[q] - kmin;
                    if ((u & mk) == lo_key && u < mn) mn = u;
                }
                lo_key = ~block_reduce<kSelThreads, true>(~mn, &sc);
            }
            lo_key += kmin;
        }
        // ---- one pass over the row; every warp lists its own candidates ----
        // A float compare against the bound's value is the same test as the key
        // compare (-0.0 compares equal to +0.0, like the keys).
        const float lo_val = key_value(lo_key);
        const float4 *s4 = reinterpret_cast<const float4 *>(srow);
        const int n4 = (n + 3) >> 2;
        const int n4full = n >> 2;
        constexpr float kNeg = -INFINITY;
        const uint32_t wlist = smem_u32(cand + wid * kCapW);
        const uint32_t lt = (1u << lane) - 1u;
        int wc = 0;  // this warp's list length (warp-uniform)
        for (int j0 = tid; j0 - tid < n4; j0 += 8 * kSelThreads) {  // uniform trip count
            float4 v[8];
            if ((j0 - tid) + 8 * kSelThreads <= n4full) {
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = __ldg(s4 + j0 + q * kSelThreads);  // 32 keys in flight
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int j4 = j0 + q * kSelThreads;
                    if (j4 < n4full) {
                        v[q] = __ldg(s4 + j4);
                    } else {  // ragged tail, element by element
                        const int e = j4 * 4;
                        v[q].x = e < n ? __ldg(srow + e) : kNeg;
                        v[q].y = e + 1 < n ? __ldg(srow + e + 1) : kNeg;
                        v[q].z = e + 2 < n ? __ldg(srow + e + 2) : kNeg;
                        v[q].w = kNeg;
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                // the four key slots of the step: their ballots order the hits of the warp
                // (slot c of every lane after slot c - 1 of every lane)
                const float x[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
                const uint32_t key0 = 4u * (uint32_t)(j0 + q * kSelThreads);
                bool hit[4];
                uint32_t bal[4];
                int cnt[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    hit[c] = x[c] >= lo_val;
                    bal[c] = __ballot_sync(0xffffffffu, hit[c]);
                    cnt[c] = __popc(bal[c]);
                }
                // a list that overflows keeps writing its last slot (the row then takes
                // the general path)
                int base = wc;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int pos = min(base + __popc(bal[c] & lt), kCapW - 1);
                    st_shared_v2_if(hit[c], wlist + 8u * (uint32_t)pos, __float_as_uint(x[c]), key0 + c);
                    base += cnt[c];
                }
                wc = base;
            }
        }
        if (lane == 0) sc.warp_cnt[wid] = wc;
        __syncthreads();
        int nc = 0;
        bool overflow = false;
#pragma unroll
        for (int w = 0; w < kSelWarps; ++w) {
            nc += sc.warp_cnt[w];
            overflow |= sc.warp_cnt[w] > kCapW;
        }
        if (!overflow && nc >= need_total) {
            // scores -> keys relative to the bound, in place (every candidate key is >= lo_key)
            uint32_t mx = 0u;
#pragma unroll 1
            for (int w = 0; w < kSelWarps; ++w) {
                const int cw = sc.warp_cnt[w];
                for (int c = tid; c < cw; c += kSelThreads) {
                    uint32_t *e = &cand[w * kCapW + c].x;
                    const uint32_t u = order_key(__uint_as_float(*e)) - lo_key;
                    *e = u;
                    mx = u > mx ? u : mx;
                }
            }
            // every candidate of every list, as (block index, relative key)
            auto each_cand = [&](auto f) {
#pragma unroll 1
                for (int w = 0; w < kSelWarps; ++w) {
                    const int cw = sc.warp_cnt[w];
                    for (int c = tid; c < cw; c += kSelThreads) {
                        const uint2 e = cand[w * kCapW + c];
                        f(e.y, e.x);
                    }
                }
            };
            const uint32_t span = block_reduce<kSelThreads, true>(mx, &sc);
            const int top = span != 0u ? 31 - __clz(span) : 0;
            // exact threshold among the listed keys (every key above it is listed)
            uint32_t prefix, mask;
            int need, in_bin;
            radix_select<kSelThreads, kCandBits>(
                [&](auto f) { each_cand([&](int, uint32_t u) { f(u); }); }, nc, need_total, top, regA, &sc,
                &prefix, &mask, &need, &in_bin);
            // a threshold value shared by more keys than slots left goes to the general
            // path (the lowest indices among them win there)
            if (need == in_bin) {
                const int nwn = (n + 31) >> 5;
                for (int w = tid; w < nwn; w += kSelThreads) regA[w] = 0u;
                __syncthreads();
                each_cand([&](uint32_t j, uint32_t u) {
                    if ((u & mask) >= prefix) atomicOr(&regA[j >> 5], 1u << (j & 31));
                });
                __syncthreads();
                // ordered emission: a block scan of the word popcounts places every winner
                emit_segment<kSelThreads>(regA, regA, nwn, 0, false, need, need_total, &out_base, &eq_base, out, &sc);
                done = true;
            }
        }
        __syncthreads();
    }

    // ============================ general path ============================
    if (!done) {
        uint32_t *gtw = regA, *eqw = regB;
        uint32_t prefix, mask;
        int need, in_bin;
        radix_select<kSelThreads, 11>(
            [&](auto f) {
                for (int j = tid; j < n; j += kSelThreads) f(order_key(__ldg(srow + j)));
            },
            n, need_total, 31, regA, &sc, &prefix, &mask, &need, &in_bin);
        const bool partial = need < in_bin;
        for (int seg0 = 0; seg0 < n; seg0 += kSegElems) {
            const int seg_n = n - seg0 < kSegElems ? n - seg0 : kSegElems;
            const int words = (seg_n + 31) >> 5;
            for (int w = wid; w < words; w += kSelWarps) {
                const int j = seg0 + w * 32 + lane;
                const bool in = j < n;
                const uint32_t u = in ? (order_key(__ldg(srow + j)) & mask) : 0u;
                const uint32_t g = __ballot_sync(0xffffffffu, in && (u > prefix || (u == prefix && !partial)));
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
            select_kernel<512><<<(unsigned)chunk, 512, sel_smem_bytes<512>(), stream>>>(
                a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, a.sel);
        else
            select_kernel<128><<<(unsigned)chunk, 128, sel_smem_bytes<128>(), stream>>>(
                a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, a.sel);
    }
    return cudaGetLastError();
}

}  // namespace qsa
