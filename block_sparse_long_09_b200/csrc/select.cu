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
// Radix passes of a select that only needs a bound of its key (a threshold below which
// no winner lies, or the bin around tau): two 8-bit digits below the keys' highest
// differing bit leave a bin of 2^-16 of their span, and stopping there saves the rest.
constexpr int kBoundPasses = 2;

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

// Query row i: its sequence *s_out and position t (decode rows, cu_q == nullptr,
// are sequence i at t = L - 1).
__device__ __forceinline__ int64_t row_position(const int32_t *cu_q, const int32_t *cu_k, int batch, int64_t i,
                                                int *s_out)
{
    if (cu_q != nullptr) {
        const int s = find_seq(cu_q, batch, i);
        *s_out = s;
        const int64_t Lq = (int64_t)cu_q[s + 1] - cu_q[s];
        const int64_t Lk = (int64_t)cu_k[s + 1] - cu_k[s];
        return (Lk - Lq) + (i - cu_q[s]);
    }
    *s_out = (int)i;
    return (int64_t)cu_k[i + 1] - cu_k[i] - 1;
}

// The selection of one row from its materialised scores srow[0 .. b_t): the own
// block b_t plus the k - 1 best, ascending, into out[0 .. k).  The whole CTA runs it.
// With nf > 1 (a multi-token decode step) the blocks bt .. bt + nf - 1 are all
// forced and the best k - nf of the candidates 0 .. bt - 1 fill the other slots.
template <int kSelThreads>
__device__ __forceinline__ void select_row(const float *__restrict__ srow, int64_t bt, int k,
                                           int32_t *__restrict__ out, uint32_t *smem_sel, SelScratch &sc,
                                           int nf = 1)
{
    constexpr int kSelWarps = kSelThreads / 32;
    constexpr int kCapW = kCandCap / kSelWarps;         // candidate list of one warp
    uint32_t *regA = smem_sel;                          // kSegWords words
    uint2 *cand = reinterpret_cast<uint2 *>(regA + kSegWords);  // kCandCap (score bits, index)
    uint32_t *regB = reinterpret_cast<uint32_t *>(cand);         // the same bytes, as words
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int need_total = k - nf;

    if (bt <= need_total) {  // every candidate fits: 0 .. b_t + nf - 1, then padding
        for (int j = tid; j < k; j += kSelThreads) out[j] = (j < bt + nf) ? j : -1;
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
        for (int f = 0; f < nf; ++f) out[need_total + f] = (int32_t)(bt + f);
    }
}

// the candidates and forced blocks of decode row s (t = L - 1) serving next_n queries
// t = L - next_n .. L - 1: candidates 0 .. b_first - 1, forced b_first .. b_last
__device__ __forceinline__ void mtp_blocks(int64_t L, int next_n, int r, int64_t *b_first, int *nf)
{
    const int64_t t_first = L - next_n > 0 ? L - next_n : 0;
    *b_first = t_first / r;
    *nf = (int)((L - 1) / r - *b_first + 1);
}

template <int kSelThreads>
__global__ void __launch_bounds__(kSelThreads, kSelThreads == 128 ? 8 : 2)
select_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ cu_q,
              const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r,
              int32_t *__restrict__ sel, int next_n)
{
    extern __shared__ uint32_t smem_sel[];
    __shared__ SelScratch sc;
    const int64_t i = row_begin + blockIdx.x;
    int s;
    const int64_t t = row_position(cu_q, cu_k, batch, i, &s);
    if (t < 0) {
        if (threadIdx.x == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        return;
    }
    int64_t bt = t / r;
    int nf = 1;
    if (next_n > 1) mtp_blocks(t + 1, next_n, r, &bt, &nf);
    if (bt > ld || bt > 0x7FFFFFFF || nf > k) {  // scores row too short for this query
        if (threadIdx.x == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        return;
    }
    select_row<kSelThreads>(scores + (int64_t)blockIdx.x * ld, bt, k, sel + i * k, smem_sel, sc, nf);
}


// ============================ fused index -> select ============================
// The prefill selection without materialised score rows (the launch order is in
// launch_index_select):
//   1. the indexer scores every stride-th kc tile of each row into a compact sample;
//   2. threshold_kernel: theta = the r_lo-th largest sample score of the row, r_lo =
//      mu + 4 sqrt(mu) + 8 with mu the expected number of the row's k - 1 winners in
//      the sample (theta = -inf where every candidate fits the candidate list);
//   3. the indexer scores every tile and appends (S, b) with S >= theta to the row's
//      candidate list (capacity cap);
//   4. select_list_kernel: the exact top k - 1 of the list.  The list holds every
//      block scoring >= theta; when it holds at least k - 1 entries and did not
//      overflow, the (k - 1)-th best is >= theta, so every block that can win, ties
//      included, is in the list and the selection equals the one over the full row.
//      Otherwise the row goes to a fallback list;
//   5. fallback_kernel: for those rows, the full score row on CUDA cores into
//      scratch, then the materialised selector.
constexpr int kThrThreads = 128;

// the compact sample row of b_t candidates: sampled tiles n = 0, stride, 2 stride, ...;
// every sample entry is valid except the tail of the last sampled tile
__device__ __forceinline__ int sample_count(int64_t bt, int stride)
{
    const int64_t tiles = (bt + 127) / 128;
    const int64_t ns_tiles = (tiles + stride - 1) / stride;
    if (ns_tiles == 0) return 0;
    const int64_t last = (ns_tiles - 1) * stride * 128;
    const int64_t tail = bt - last < 128 ? bt - last : 128;
    return (int)((ns_tiles - 1) * 128 + tail);
}

__global__ void __launch_bounds__(kThrThreads)
threshold_kernel(const float *__restrict__ sample, int64_t sample_ld, int stride, const int32_t *__restrict__ cu_q,
                 const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r, int list_cap,
                 float *__restrict__ theta, int32_t *__restrict__ fb_count)
{
    extern __shared__ uint32_t smem_sel[];
    uint32_t *hist = smem_sel;            // kSegWords words
    uint32_t *keys = smem_sel + kSegWords;  // sample_ld words
    __shared__ SelScratch sc;
    const int tid = threadIdx.x;
    if (blockIdx.x == 0 && tid == 0) *fb_count = 0;  // the fallback list of this call starts empty
    const int64_t rl = blockIdx.x, i = row_begin + rl;
    int s;
    const int64_t t = row_position(cu_q, cu_k, batch, i, &s);
    const int64_t bt = t >= 0 ? t / r : 0;
    if (bt <= list_cap) {  // every candidate fits the list
        if (tid == 0) theta[rl] = -INFINITY;
        return;
    }
    const int ns = sample_count(bt, stride);
    const float mu = (float)(k - 1) * (float)ns / (float)bt;
    const int r_lo = (int)ceilf(mu + 4.f * sqrtf(mu) + 8.f);
    if (ns > sample_ld || r_lo > ns) {  // no usable sample: collect everything (the fallback takes it)
        if (tid == 0) theta[rl] = -INFINITY;
        return;
    }
    const float *srow = sample + rl * sample_ld;
    // keys relative to the sample's smallest: the radix starts at their highest differing bit
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int p = tid; p < ns; p += kThrThreads) {
        const uint32_t u = order_key(__ldg(srow + p));
        keys[p] = u;
        kmin = min(kmin, u);
        kmax = max(kmax, u);
    }
    kmin = ~kmin;
    block_max2<kThrThreads>(kmin, kmax, &sc);  // (its barrier also publishes keys[])
    kmin = ~kmin;
    const uint32_t span = kmax - kmin;
    uint32_t prefix, mask;
    int need, in_bin;
    radix_select<kThrThreads, 8>(
        [&](auto f) {
            for (int p = tid; p < ns; p += kThrThreads) f(keys[p] - kmin);
        },
        ns, r_lo, span != 0u ? 31 - __clz(span) : 0, hist, &sc, &prefix, &mask, &need, &in_bin, kBoundPasses);
    // prefix + kmin is the r_lo-th largest key, or (bin taken whole, or the passes spent) a
    // lower bound of it
    if (tid == 0) theta[rl] = key_value(prefix + kmin);
}

// The exact top k - 1 of a candidate list (order key, block index) in shared
// memory that holds every block able to win, ascending into out[0 .. k), with
// out[k - 1] = b_t.  Ties at the threshold value go to the lowest block indices.
template <int kT>
__device__ __forceinline__ void select_from_list(const uint2 *cand, int cnt, int64_t bt, int k,
                                                 int32_t *__restrict__ out, uint32_t *regA, SelScratch &sc,
                                                 int nf = 1)
{
    const int tid = threadIdx.x;
    const int need_total = k - nf;
    // keys relative to the list's smallest, so the radix starts at their highest differing bit
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int c = tid; c < cnt; c += kT) {
        kmin = min(kmin, cand[c].x);
        kmax = max(kmax, cand[c].x);
    }
    kmin = ~kmin;
    block_max2<kT>(kmin, kmax, &sc);
    kmin = ~kmin;
    const uint32_t span = cnt > 0 ? kmax - kmin : 0u;
    uint32_t prefix, mask;
    int need, in_bin;
    radix_select<kT, 8>(
        [&](auto f) {
            for (int c = tid; c < cnt; c += kT) f(cand[c].x - kmin);
        },
        cnt, need_total, span != 0u ? 31 - __clz(span) : 0, regA, &sc, &prefix, &mask, &need, &in_bin);
    // winners: keys above the threshold bin, and of the bin either all (need == in_bin) or,
    // when the exact threshold value has more entries than slots left, its lowest indices
    uint32_t iprefix = 0u, imask = 0u;
    const bool partial = need < in_bin;
    if (partial) {
        int n2, b2;
        radix_select<kT, 8>(
            [&](auto f) {
                for (int c = tid; c < cnt; c += kT)
                    if (((cand[c].x - kmin) & mask) == prefix) f(~cand[c].y);
            },
            in_bin, need, 31, regA, &sc, &iprefix, &imask, &n2, &b2);
    }
    auto wins = [&](const uint2 e) -> bool {
        const uint32_t u = (e.x - kmin) & mask;
        if (u != prefix) return u > prefix;
        return !partial || ((~e.y) & imask) >= iprefix;
    };
    // ordered emission, one 65536-block segment of the bitmap at a time
    int out_base = 0, eq_base = 0;
    for (int64_t seg0 = 0; seg0 < bt; seg0 += kSegElems) {
        const int seg_n = (int)(bt - seg0 < kSegElems ? bt - seg0 : kSegElems);
        const int words = (seg_n + 31) >> 5;
        for (int wd = tid; wd < words; wd += kT) regA[wd] = 0u;
        __syncthreads();
        for (int c = tid; c < cnt; c += kT) {
            const uint2 e = cand[c];
            const int64_t b = (int64_t)e.y - seg0;
            if (b >= 0 && b < seg_n && wins(e)) atomicOr(&regA[b >> 5], 1u << (b & 31));
        }
        __syncthreads();
        emit_segment<kT>(regA, regA, words, (int)seg0, false, need_total, need_total, &out_base, &eq_base,
                                  out, &sc);
        __syncthreads();
    }
    if (tid == 0) {
        if (out_base != need_total) set_device_status(QSA_ERR_DEVICE_CHECK);
        for (int f = 0; f < nf; ++f) out[need_total + f] = (int32_t)(bt + f);
    }
}

__global__ void __launch_bounds__(kThrThreads, 8)
select_list_kernel(const uint2 *__restrict__ lists, const int32_t *__restrict__ counts, int list_cap,
                   const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k, int batch, int64_t row_begin,
                   int k, int r, int32_t *__restrict__ sel, int32_t *__restrict__ fb_count,
                   int32_t *__restrict__ fb_rows)
{
    extern __shared__ uint32_t smem_sel[];
    uint32_t *regA = smem_sel;                                   // kSegWords words
    uint2 *cand = reinterpret_cast<uint2 *>(smem_sel + kSegWords);  // list_cap (key, index)
    __shared__ SelScratch sc;
    const int tid = threadIdx.x;
    const int64_t rl = blockIdx.x, i = row_begin + rl;
    int s;
    const int64_t t = row_position(cu_q, cu_k, batch, i, &s);
    if (t < 0) {
        if (tid == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        return;
    }
    const int64_t bt = t / r;
    int32_t *out = sel + i * k;
    const int need_total = k - 1;
    if (bt <= need_total) {
        for (int j = tid; j < k; j += kThrThreads) out[j] = (j <= bt) ? j : -1;
        return;
    }
    // the row's list is 4 segments of list_cap / 4 entries (one per TMEM lane quadrant
    // of the indexer), each with its own length
    const int cap_q = list_cap / 4;
    const int4 c4 = *reinterpret_cast<const int4 *>(counts + rl * 4);
    const int cq[4] = {c4.x, c4.y, c4.z, c4.w};
    const int cnt = cq[0] + cq[1] + cq[2] + cq[3];
    if (cnt < need_total || cq[0] > cap_q || cq[1] > cap_q || cq[2] > cap_q || cq[3] > cap_q) {
        // the bound was too high, or a segment overflowed
        if (tid == 0) fb_rows[atomicAdd(fb_count, 1)] = (int32_t)rl;
        return;
    }
    const uint2 *lrow = lists + rl * list_cap;
    int off = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        for (int c = tid; c < cq[q]; c += kThrThreads) {
            const uint2 e = lrow[q * cap_q + c];
            cand[off + c] = make_uint2(order_key(__uint_as_float(e.x)), e.y);
        }
        off += cq[q];
    }
    __syncthreads();
    select_from_list<kThrThreads>(cand, cnt, bt, k, out, regA, sc);
}

constexpr int kFbThreads = 512;

__global__ void __launch_bounds__(kFbThreads, 1)
fallback_kernel(const __nv_bfloat16 *__restrict__ q_idx, const float *__restrict__ w, const __nv_bfloat16 *__restrict__ kc,
                const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                const int32_t *__restrict__ cu_blocks, int batch, int64_t row_begin, int k, int r,
                const int32_t *__restrict__ fb_count, const int32_t *__restrict__ fb_rows, float *__restrict__ scratch,
                int64_t scratch_ld, int32_t *__restrict__ sel, int next_n)
{
    pdl_enter();
    extern __shared__ uint32_t smem_sel[];
    __shared__ SelScratch sc;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = *fb_count;
    float *srow = scratch + (int64_t)blockIdx.x * scratch_ld;
    for (int f = blockIdx.x; f < n; f += gridDim.x) {
        const int64_t i = row_begin + fb_rows[f];
        int s;
        const int64_t t = row_position(cu_q, cu_k, batch, i, &s);
        int64_t bt = t / r;
        int nf = 1;
        if (next_n > 1) mtp_blocks(t + 1, next_n, r, &bt, &nf);
        if (bt > scratch_ld || nf > k) {
            if (threadIdx.x == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
            continue;
        }
        index_row_cuda<2>(q_idx + i * 512, w + i * 4, kc + (int64_t)cu_blocks[s] * 256, 0, bt, srow, warp,
                       kFbThreads / 32, lane);
        __syncthreads();
        select_row<kFbThreads>(srow, bt, k, sel + i * k, smem_sel, sc, nf);
        __syncthreads();
    }
}

// ============================ decode: hi-plane scan, then refine ============================
// The decode indexer reads only the hi plane of the compressed keys (half the
// bytes of the exact hi + lo scan).  With the RMSNorm, ||kc_b|| <= sqrt(d), and
// the lo plane is the rounding residue of the hi plane, ||lo_b|| <= 2^-8 ||kc_b||;
// a head's dot moves by at most ||q_h|| ||lo_b||, ReLU is 1-Lipschitz, so every
// approximate score is within E = sum_h |w_h| ||q_h|| sqrt(d) (2^-8 1.01 + 1e-4) of
// the exact one (the last term covers fp32 accumulation).  Per row:
//   1. tau = the (k-1)-th largest approximate score (radix select over the row);
//   2. the window W = {b : approx_b >= tau - 2E} holds every block that can win:
//      at least k - 1 blocks have approx >= tau, so exact >= tau - E for them,
//      while a block outside W has exact < tau - E;
//   3. the blocks of W are rescored exactly (hi + lo planes, the same arithmetic
//      as the exact decode indexer) and their exact top k - 1 is the selection.
// A window larger than kRefCap goes to the fallback (exact scores of the whole row).
constexpr int kRefThreads = 512;
constexpr int kRefCap = 4096;
constexpr int kRefSmem = kSegWords * 4 + kRefCap * (8 + 4 + 4);

// E of a decode row (called by one warp; every lane returns it): the head dots move by at
// most ||q_h|| ||lo_b|| with ||lo_b|| <= 2^-8 ||kc_b|| = 2^-8 sqrt(128)
__device__ __forceinline__ float row_error_bound(const __nv_bfloat16 *__restrict__ q_row,
                                                 const float *__restrict__ w_row, int lane)
{
    float e = 0.f;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(q_row + h * 128 + lane * 4);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
        float ss = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        e += fabsf(__ldg(w_row + h)) * sqrtf(ss);
    }
    return e * 11.3137085f * (1.01f * 0.00390625f + 1e-4f) * 1.01f;  // sqrt(128) (2^-8 1.01 + 1e-4)
}

// theta_s, a lower bound of tau (the (k-1)-th largest of the n > kRefCap approximate
// scores srow[0 .. n)): the r_lo-th largest of a sample of the row (runs of 8 keys spread
// over it), r_lo = mu + 4 sqrt(mu) + 8 for mu expected winners in the sample.  The whole
// CTA calls it; every thread returns theta_s.  skeys: 8192 words of shared memory.
__device__ __forceinline__ float sample_bound(const float *__restrict__ srow, int n, int need_total,
                                              uint32_t *skeys, uint32_t *hist, SelScratch &sc)
{
    const int tid = threadIdx.x;
    // about n / 32 keys (runs of 8, at least 2048, at most 8192): some 16 expected winners
    // fall in the sample, so the bound stays tight on long rows (with 2048 keys a
    // 262143-block row keeps only 4, and its list overflows); every run starts at least
    // 16 keys before the row's end
    int runs = n / 256;
    runs = runs < kCandCap / 8 ? kCandCap / 8 : (runs > kRefCap / 4 ? kRefCap / 4 : runs);
    const int ns = runs * 8;
    for (int g = tid; g < runs; g += kRefThreads) {
        const int at = (int)(((int64_t)g * n) / runs) & ~3;
        const float4 x0 = __ldg(reinterpret_cast<const float4 *>(srow + at));
        const float4 x1 = __ldg(reinterpret_cast<const float4 *>(srow + at + 4));
        const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) skeys[g * 8 + e] = order_key(xs[e]);
    }
    __syncthreads();
    const float mu = (float)need_total * (float)ns / (float)n;
    int r_lo = (int)ceilf(mu + 4.f * sqrtf(mu) + 8.f);
    if (r_lo > ns) r_lo = ns;
    // keys relative to the sample's smallest: the radix starts at their highest differing bit
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int q = tid; q < ns; q += kRefThreads) {
        kmin = min(kmin, skeys[q]);
        kmax = max(kmax, skeys[q]);
    }
    kmin = ~kmin;
    block_max2<kRefThreads>(kmin, kmax, &sc);
    kmin = ~kmin;
    const uint32_t span = kmax - kmin;
    uint32_t sp, sm;
    int sn, sb;
    radix_select<kRefThreads, 8>(
        [&](auto f) {
            for (int q = tid; q < ns; q += kRefThreads) f(skeys[q] - kmin);
        },
        ns, r_lo, span != 0u ? 31 - __clz(span) : 0, hist, &sc, &sp, &sm, &sn, &sb, kBoundPasses);
    return key_value(sp + kmin);  // the sample's r_lo-th largest, or its bin's floor
}

// The decode row's position and the counts of its selection (k - nf slots for the best
// candidates 0 .. bt - 1); false when the row is not a valid decode row.
__device__ __forceinline__ bool refine_row(const int32_t *cu_q, const int32_t *cu_k, int batch, int64_t i, int r,
                                           int next_n, int64_t ld, int k, int *s, int64_t *bt, int *nf)
{
    const int64_t t = row_position(cu_q, cu_k, batch, i, s);
    if (t < 0) return false;
    *bt = t / r;
    *nf = 1;
    if (next_n > 1) mtp_blocks(t + 1, next_n, r, bt, nf);
    return !(*bt > ld || *bt > 0x7FFFFFFF || *nf > k);
}

// Batches too small to fill the GPU with one refine CTA per row build the candidate
// lists W' in two launches before the refine: refine_bound_kernel (E and theta_s per
// row, the list counter reset) and refine_list_kernel (CTAs over (row chunk, row) append
// the approximate scores >= theta_s - 2E to the row's list in global memory).
constexpr int kListChunk = 4096;  // approximate scores scanned by one list CTA
constexpr int kListThreads = 256;
constexpr int kBoundSmem = (kSegWords + 2 * kRefCap) * 4;

__global__ void __launch_bounds__(kRefThreads, 1)
refine_bound_kernel(const float *__restrict__ approx, int64_t ld, const __nv_bfloat16 *__restrict__ q_idx,
                    const float *__restrict__ w, const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                    int batch, int64_t row_begin, int k, int r, int next_n, float2 *__restrict__ bound,
                    int32_t *__restrict__ count)
{
    pdl_enter();
    extern __shared__ uint32_t smem_sel[];
    __shared__ SelScratch sc;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rl = blockIdx.x, i = row_begin + rl;
    if (tid == 0) count[rl] = 0;
    int s, nf;
    int64_t bt;
    if (!refine_row(cu_q, cu_k, batch, i, r, next_n, ld, k, &s, &bt, &nf)) return;  // the refine flags it
    const int need_total = k - nf;
    if (bt <= need_total) return;  // every candidate wins: the refine writes it
    const int n = (int)bt;
    float theta_s = -INFINITY;
    if (n > kRefCap) theta_s = sample_bound(approx + rl * ld, n, need_total, smem_sel + kSegWords, smem_sel, sc);
    if (warp == 0) {
        const float e = row_error_bound(q_idx + i * 512, w + i * 4, lane);
        if (lane == 0) bound[rl] = make_float2(theta_s, e);
    }
}

__global__ void __launch_bounds__(kListThreads)
refine_list_kernel(const float *__restrict__ approx, int64_t ld, const int32_t *__restrict__ cu_q,
                   const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r, int next_n,
                   const float2 *__restrict__ bound, uint2 *__restrict__ lists, int32_t *__restrict__ count)
{
    pdl_enter();
    constexpr int kW = kListThreads / 32, kPer = kListChunk / (4 * kListThreads);  // float4 groups per thread
    __shared__ int warp_hits[kW];
    __shared__ int cta_base;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rl = blockIdx.y, i = row_begin + rl;
    int s, nf;
    int64_t bt;
    if (!refine_row(cu_q, cu_k, batch, i, r, next_n, ld, k, &s, &bt, &nf)) return;  // uniform per CTA
    if (bt <= k - nf) return;
    const int n = (int)bt;
    const int c0 = blockIdx.x * kListChunk;
    if (c0 >= n) return;
    const float2 b = bound[rl];
    const float lo_bound = b.x - 2.f * b.y;
    const float4 *srow4 = reinterpret_cast<const float4 *>(approx + rl * ld + c0);
    const int len = n - c0 < kListChunk ? n - c0 : kListChunk;
    const int n4 = (len + 3) / 4;
    float4 x4[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int g = u * kListThreads + tid;
        x4[u] = g < n4 ? __ldg(srow4 + g) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    uint32_t m[kPer * 4];
    int hits = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int g = u * kListThreads + tid;
        const float xs[4] = {x4[u].x, x4[u].y, x4[u].z, x4[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            m[u * 4 + e] = __ballot_sync(0xffffffffu, 4 * g + e < len && xs[e] >= lo_bound);
            hits += __popc(m[u * 4 + e]);
        }
    }
    // one reservation of list slots per CTA: the warps' counts, their prefix, one atomic
    if (lane == 0) warp_hits[warp] = hits;
    __syncthreads();
    if (tid == 0) {
        int tot = 0;
        for (int x = 0; x < kW; ++x) {
            const int h = warp_hits[x];
            warp_hits[x] = tot;
            tot += h;
        }
        cta_base = tot > 0 ? atomicAdd(count + rl, tot) : 0;
    }
    __syncthreads();
    if (hits == 0) return;  // warp-uniform
    int base = cta_base + warp_hits[warp];
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint2 *lrow = lists + rl * kRefCap;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int g = u * kListThreads + tid;
        const float xs[4] = {x4[u].x, x4[u].y, x4[u].z, x4[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t mk = m[u * 4 + e];
            const int pos = base + __popc(mk & lt_mask);
            if (((mk >> lane) & 1u) && pos < kRefCap) lrow[pos] = make_uint2(order_key(xs[e]), (uint32_t)(c0 + 4 * g + e));
            base += __popc(mk);
        }
    }
}

template <bool kListed>
__global__ void __launch_bounds__(kRefThreads, 1)
refine_select_kernel(const float *__restrict__ approx, int64_t ld, const __nv_bfloat16 *__restrict__ q_idx,
                     const float *__restrict__ w, const __nv_bfloat16 *__restrict__ kc,
                     const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k,
                     const int32_t *__restrict__ cu_blocks, int batch, int64_t row_begin, int k, int r,
                     int32_t *__restrict__ sel, int32_t *__restrict__ fb_count, int32_t *__restrict__ fb_rows,
                     int next_n, const float2 *__restrict__ bound, const uint2 *__restrict__ lists,
                     const int32_t *__restrict__ count)
{
    pdl_enter();
    extern __shared__ uint32_t smem_sel[];
    uint32_t *regA = smem_sel;                                        // kSegWords words
    uint2 *cand = reinterpret_cast<uint2 *>(smem_sel + kSegWords);    // kRefCap (key, index)
    float *exact = reinterpret_cast<float *>(cand + kRefCap);         // kRefCap exact scores
    int32_t *widx = reinterpret_cast<int32_t *>(exact + kRefCap);     // kRefCap window block ids
    __shared__ SelScratch sc;
    __shared__ int wcount;
    __shared__ float e_row;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rl = blockIdx.x, i = row_begin + rl;
    int s, nf;
    int64_t bt;
    if (!refine_row(cu_q, cu_k, batch, i, r, next_n, ld, k, &s, &bt, &nf)) {
        if (tid == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        return;
    }
    int32_t *out = sel + i * k;
    const int need_total = k - nf;
    if (bt <= need_total) {
        for (int j = tid; j < k; j += kRefThreads) out[j] = (j < bt + nf) ? j : -1;
        return;
    }
    const int n = (int)bt;
    const uint32_t lt_mask = (1u << lane) - 1u;
    float theta_s = -INFINITY;
    if constexpr (kListed) {
        // the bound and the list W' come from refine_bound_kernel and refine_list_kernel
        const float2 b = bound[rl];
        theta_s = b.x;
        if (tid == 0) {
            e_row = b.y;
            wcount = __ldcg(count + rl);
        }
        __syncthreads();
        const int cnt = wcount;
        if (cnt <= kRefCap)
            for (int c = tid; c < cnt; c += kRefThreads) cand[c] = __ldcg(lists + rl * kRefCap + c);
    } else {
        const float *srow = approx + rl * ld;
        // the error bound E of the row
        if (warp == 0) {
            const float e = row_error_bound(q_idx + i * 512, w + i * 4, lane);
            if (lane == 0) {
                e_row = e;
                wcount = 0;
            }
        }
        // 1. a lower bound theta_s of tau, the (k-1)-th largest approximate score, from a
        //    sample; every block when the row fits the list
        if (n > kRefCap) theta_s = sample_bound(srow, n, need_total, reinterpret_cast<uint32_t *>(cand), regA, sc);
        __syncthreads();
        // 2. the candidates W' = {b : approx_b >= theta_s - 2E} (with their approximate keys)
        const float lo_bound = theta_s - 2.f * e_row;
        // rows are 16-byte aligned with ld a multiple of 4: float4 groups, kRefUnroll of
        // them in flight per thread; keys past n (inside the last group) are masked
        constexpr int kRefUnroll = 4;
        const int n4 = (n + 3) / 4;
        const float4 *srow4 = reinterpret_cast<const float4 *>(srow);
        for (int g0 = 0; g0 < n4; g0 += kRefThreads * kRefUnroll) {
            float4 x4[kRefUnroll];
#pragma unroll
            for (int u = 0; u < kRefUnroll; ++u) {
                const int g = g0 + u * kRefThreads + tid;
                x4[u] = g < n4 ? __ldg(srow4 + g) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            }
            // the warp's hits of the whole batch take one reservation of list slots
            uint32_t m[kRefUnroll * 4];
            int total = 0;
#pragma unroll
            for (int u = 0; u < kRefUnroll; ++u) {
                const int g = g0 + u * kRefThreads + tid;
                const float xs[4] = {x4[u].x, x4[u].y, x4[u].z, x4[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    m[u * 4 + e] = __ballot_sync(0xffffffffu, 4 * g + e < n && xs[e] >= lo_bound);
                    total += __popc(m[u * 4 + e]);
                }
            }
            if (total == 0) continue;  // warp-uniform
            int base = 0;
            if (lane == 0) base = atomicAdd(&wcount, total);
            base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
            for (int u = 0; u < kRefUnroll; ++u) {
                const int g = g0 + u * kRefThreads + tid;
                const float xs[4] = {x4[u].x, x4[u].y, x4[u].z, x4[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t mk = m[u * 4 + e];
                    const int pos = base + __popc(mk & lt_mask);
                    if (((mk >> lane) & 1u) && pos < kRefCap) cand[pos] = make_uint2(order_key(xs[e]), (uint32_t)(4 * g + e));
                    base += __popc(mk);
                }
            }
        }
    }
    __syncthreads();
    int nw = wcount;
    if (nw > kRefCap || nw < need_total) {  // the list does not fit, or the bound was too high
        if (tid == 0) fb_rows[atomicAdd(fb_count, 1)] = (int32_t)rl;
        return;
    }
    //    tau among them (every key >= tau is listed when at least k - 1 keys are >= theta_s)
    const uint32_t ks = order_key(theta_s);
    int above = 0;
    for (int c = tid; c < nw; c += kRefThreads) above += cand[c].x >= ks ? 1 : 0;
    above = (int)block_reduce<kRefThreads, false>((uint32_t)above, &sc);
    if (above < need_total) {
        if (tid == 0) fb_rows[atomicAdd(fb_count, 1)] = (int32_t)rl;
        return;
    }
    uint32_t prefix, mask, tau_hi;
    int need, in_bin;
    {
        uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
        for (int c = tid; c < nw; c += kRefThreads) {
            kmin = min(kmin, cand[c].x);
            kmax = max(kmax, cand[c].x);
        }
        kmin = ~kmin;
        block_max2<kRefThreads>(kmin, kmax, &sc);
        kmin = ~kmin;
        const uint32_t span = kmax - kmin;
        radix_select<kRefThreads, 8>(
            [&](auto f) {
                for (int c = tid; c < nw; c += kRefThreads) f(cand[c].x - kmin);
            },
            nw, need_total, span != 0u ? 31 - __clz(span) : 0, regA, &sc, &prefix, &mask, &need, &in_bin,
            kBoundPasses);
        tau_hi = min(prefix | ~mask, span) + kmin;  // the bin's largest key: an upper bound of tau
        prefix += kmin;                             // tau (or its bin's floor, a lower bound) as an absolute key
    }
    //    the window W = {b : approx_b >= tau - 2E}.  tau_exact, the exact (k-1)-th best,
    //    lies in [tau - E, tau + E] (k - 1 blocks have approx >= tau, at most k - 2 have
    //    approx > tau), so a block with approx > tau + 2E has exact > tau_exact: a certain
    //    winner, not rescored.  The band's block ids are compacted from the front of widx,
    //    the certain winners' from the back.
    const uint32_t kw = order_key(key_value(prefix) - 2.f * e_row);
    const uint32_t kw_hi = order_key(key_value(tau_hi) + 2.f * e_row);
    __shared__ int ccount;
    if (tid == 0) {
        wcount = 0;
        ccount = 0;
    }
    __syncthreads();
    for (int c0 = 0; c0 < nw; c0 += kRefThreads) {
        const int c = c0 + tid;
        const uint32_t key = c < nw ? cand[c].x : 0u;
        const bool sure = c < nw && key > kw_hi;
        const bool band = c < nw && !sure && key >= kw;
        const uint32_t mb = __ballot_sync(0xffffffffu, band), ms = __ballot_sync(0xffffffffu, sure);
        int bb = 0, bs = 0;
        if (lane == 0 && mb != 0u) bb = atomicAdd(&wcount, __popc(mb));
        if (lane == 0 && ms != 0u) bs = atomicAdd(&ccount, __popc(ms));
        bb = __shfl_sync(0xffffffffu, bb, 0);
        bs = __shfl_sync(0xffffffffu, bs, 0);
        if (band) widx[bb + __popc(mb & lt_mask)] = (int32_t)cand[c].y;
        if (sure) widx[kRefCap - 1 - (bs + __popc(ms & lt_mask))] = (int32_t)cand[c].y;
    }
    __syncthreads();
    const int nb = wcount, ncs = ccount;
    // 3. exact scores of the band, then the exact top k - 1 of band and certain winners
    //    (these with the largest key, which no finite score reaches)
    const __nv_bfloat16 *kc_seq = kc + (int64_t)cu_blocks[s] * 256;
    index_row_cuda_at<2>(q_idx + i * 512, w + i * 4,
                         [=](int64_t p) { return kc_seq + (int64_t)widx[p] * 256; }, 0, nb, exact, warp,
                         kRefThreads / 32, lane);
    __syncthreads();
    for (int c = tid; c < nb; c += kRefThreads) cand[c] = make_uint2(order_key(exact[c]), (uint32_t)widx[c]);
    for (int c = tid; c < ncs; c += kRefThreads) cand[nb + c] = make_uint2(0xFFFFFFFFu, (uint32_t)widx[kRefCap - 1 - c]);
    __syncthreads();
    select_from_list<kRefThreads>(cand, nb + ncs, bt, k, out, regA, sc, nf);
}

__global__ void clear_count_kernel(int32_t *c)
{
    pdl_enter();
    *c = 0;
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
                a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, a.sel, a.next_n);
        else
            select_kernel<128><<<(unsigned)chunk, 128, sel_smem_bytes<128>(), stream>>>(
                a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, a.sel, a.next_n);
    }
    return cudaGetLastError();
}


size_t index_select_workspace_bytes(int64_t rows, int64_t max_len_k, int k, int r, int grid)
{
    const IndexSelectLayout L = index_select_layout(rows, max_len_k, k, r, grid);
    return L.total;
}

IndexSelectLayout index_select_layout(int64_t rows, int64_t max_len_k, int k, int r, int grid)
{
    IndexSelectLayout L{};
    const int64_t max_bt = max_len_k > 0 ? (max_len_k - 1) / r : 0;
    const int64_t tiles = (max_bt + 127) / 128;
    L.list_cap = 4 * k;
    L.stride = 16;
    // at most 8192 sample entries per row (32 KB of keys for the threshold kernel)
    while ((tiles + L.stride - 1) / L.stride > 64) L.stride *= 2;
    L.sample_ld = ((tiles + L.stride - 1) / L.stride) * 128;
    if (L.sample_ld == 0) L.sample_ld = 128;
    L.scratch_ld = (max_bt + 3) / 4 * 4 + 4;
    L.grid = grid;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t off = 0;
    L.off_sample = off; off = al(off + (size_t)rows * L.sample_ld * 4);
    L.off_theta = off; off = al(off + (size_t)rows * 4);
    L.off_counts = off; off = al(off + (size_t)rows * 4 * 4);  // 4 list segments per row
    L.off_lists = off; off = al(off + (size_t)rows * L.list_cap * 8);
    L.off_fb = off; off = al(off + (size_t)(rows + 1) * 4);
    L.off_scratch = off; off = al(off + (size_t)grid * L.scratch_ld * 4);
    L.total = off;
    return L;
}

cudaError_t launch_index_select(const IndexArgs &a, int k, void *ws, int grid, int64_t max_len_k, int32_t *sel,
                                cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0) return cudaSuccess;
    if (rows > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const IndexSelectLayout L = index_select_layout(rows, max_len_k, k, a.r, grid);
    uint8_t *base = static_cast<uint8_t *>(ws);
    float *sample = reinterpret_cast<float *>(base + L.off_sample);
    float *theta = reinterpret_cast<float *>(base + L.off_theta);
    int32_t *counts = reinterpret_cast<int32_t *>(base + L.off_counts);
    uint2 *lists = reinterpret_cast<uint2 *>(base + L.off_lists);
    int32_t *fb_count = reinterpret_cast<int32_t *>(base + L.off_fb);
    int32_t *fb_rows = fb_count + 1;
    float *scratch = reinterpret_cast<float *>(base + L.off_scratch);
    cudaError_t e;
    // 1. sample scores (rows whose candidates all fit the list are skipped)
    IdxOut o1{};
    o1.mode = 1;
    o1.sample = sample;
    o1.sample_ld = L.sample_ld;
    o1.stride = L.stride;
    o1.min_bt = L.list_cap;
    if ((e = launch_index_tc_mode(a, o1, stream)) != cudaSuccess) return e;
    // 2. thresholds (also clears the fallback count)
    threshold_kernel<<<(unsigned)rows, kThrThreads, (kSegWords + (int)L.sample_ld) * 4, stream>>>(
        sample, L.sample_ld, L.stride, a.cu_q, a.cu_k, a.batch, a.row_begin, k, a.r, L.list_cap, theta, fb_count);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. candidate lists
    IdxOut o3{};
    o3.mode = 2;
    o3.theta = theta;
    o3.lists = lists;
    o3.list_cap = L.list_cap;
    o3.counts = counts;
    if ((e = launch_index_tc_mode(a, o3, stream)) != cudaSuccess) return e;
    // 4. exact selection over each list
    const int smem4 = (kSegWords + 2 * L.list_cap) * 4;
    if ((e = set_smem_attr_once(reinterpret_cast<const void *>(select_list_kernel), smem4)) != cudaSuccess) return e;
    select_list_kernel<<<(unsigned)rows, kThrThreads, smem4, stream>>>(
        lists, counts, L.list_cap, a.cu_q, a.cu_k, a.batch, a.row_begin, k, a.r, sel, fb_count, fb_rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 5. fallback rows
    fallback_kernel<<<(unsigned)L.grid, kFbThreads, sel_smem_bytes<kFbThreads>(), stream>>>(
        a.q_idx, a.w, a.kc, a.cu_q, a.cu_k, a.cu_blocks, a.batch, a.row_begin, k, a.r, fb_count, fb_rows, scratch,
        L.scratch_ld, sel, 1);
    return cudaGetLastError();
}

// Below this many rows the candidate lists are built by their own launches (most SMs
// would otherwise idle while one CTA per row scans its row).
constexpr int64_t kListedRows = 32;

size_t decode_select_workspace_bytes(int64_t rows, int64_t ld, int grid)
{
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    // approximate scores, fallback rows, fallback scratch, then the listed path's bounds,
    // list counters and lists
    return al((size_t)rows * ld * 4) + al((size_t)(rows + 1) * 4) + al((size_t)grid * ld * 4) +
           al((size_t)rows * 8) + al((size_t)rows * 4) + al((size_t)rows * kRefCap * 8);
}

cudaError_t launch_decode_index_select(const IndexArgs &a, int k, void *ws, int grid, bool refine, int32_t *sel,
                                       cudaStream_t stream, int next_n)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0) return cudaSuccess;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    uint8_t *base = static_cast<uint8_t *>(ws);
    size_t off = 0;
    float *scores = reinterpret_cast<float *>(base);
    off += al((size_t)rows * a.ld * 4);
    int32_t *fb_count = reinterpret_cast<int32_t *>(base + off);
    int32_t *fb_rows = fb_count + 1;
    off += al((size_t)(rows + 1) * 4);
    float *scratch = reinterpret_cast<float *>(base + off);
    off += al((size_t)grid * a.ld * 4);
    float2 *bound = reinterpret_cast<float2 *>(base + off);
    off += al((size_t)rows * 8);
    int32_t *count = reinterpret_cast<int32_t *>(base + off);
    off += al((size_t)rows * 4);
    uint2 *lists = reinterpret_cast<uint2 *>(base + off);
    IndexArgs a2 = a;
    a2.scores = scores;
    cudaError_t e;
    if (!refine) {  // exact scores (hi + lo), then the selector
        if ((e = launch_index_rowwise(a2, stream)) != cudaSuccess) return e;
        SelectArgs sa{scores, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin, a.row_end, sel, k, a.r};
        sa.next_n = next_n;
        return launch_select(sa, stream);
    }
    if ((e = launch_index_rowwise_hi(a2, stream)) != cudaSuccess) return e;
    if ((e = launch_pdl(clear_count_kernel, dim3(1), dim3(1), 0, stream, fb_count)) != cudaSuccess) return e;
    if (rows > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const bool listed = rows < kListedRows;
    if (listed) {
        if ((e = set_smem_attr_once(reinterpret_cast<const void *>(refine_bound_kernel), kBoundSmem)) != cudaSuccess)
            return e;
        if ((e = launch_pdl(refine_bound_kernel, dim3((unsigned)rows), dim3(kRefThreads), kBoundSmem, stream,
                            (const float *)scores, a.ld, a.q_idx, a.w, a.cu_q, a.cu_k, a.batch, a.row_begin, k, a.r,
                            next_n, bound, count)) != cudaSuccess)
            return e;
        const int64_t chunks = (a.ld + kListChunk - 1) / kListChunk;
        if (chunks > 0x7FFFFFFF || rows > 65535) return cudaErrorInvalidValue;
        if ((e = launch_pdl(refine_list_kernel, dim3((unsigned)chunks, (unsigned)rows), dim3(kListThreads), 0, stream,
                            (const float *)scores, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin, k, a.r, next_n,
                            (const float2 *)bound, lists, count)) != cudaSuccess)
            return e;
    }
    auto kern = listed ? refine_select_kernel<true> : refine_select_kernel<false>;
    if ((e = set_smem_attr_once(reinterpret_cast<const void *>(kern), kRefSmem)) != cudaSuccess) return e;
    if ((e = launch_pdl(kern, dim3((unsigned)rows), dim3(kRefThreads), kRefSmem, stream, (const float *)scores, a.ld,
                        a.q_idx, a.w, a.kc, a.cu_q, a.cu_k, a.cu_blocks, a.batch, a.row_begin, k, a.r, sel, fb_count,
                        fb_rows, next_n, (const float2 *)bound, (const uint2 *)lists, (const int32_t *)count)) !=
        cudaSuccess)
        return e;
    return launch_pdl(fallback_kernel, dim3((unsigned)grid), dim3(kFbThreads), sel_smem_bytes<kFbThreads>(), stream,
                      a.q_idx, a.w, a.kc, a.cu_q, a.cu_k, a.cu_blocks, a.batch, a.row_begin, k, a.r,
                      (const int32_t *)fb_count, (const int32_t *)fb_rows, scratch, a.ld, sel, next_n);
}

}  // namespace qsa
