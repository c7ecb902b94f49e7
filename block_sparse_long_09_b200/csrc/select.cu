// select.cu -- QSA top-k micro-block selection.
//
// Budget sentence of "On the Design of Qwen3.8 Next Architecture" (reading
// notes, section 6): per query, the own (trailing, possibly incomplete) causal
// block b_t is always kept and the remaining k - 1 slots go to the best complete
// blocks 0 .. b_t - 1.  Ties go to the lower block index; the output lists the
// chosen blocks in ascending order, padded with -1.
//
// One CTA (512 threads) per query row.  The fp32 scores become order-preserving
// 32-bit keys (sign-flip trick, -0.0 folded into +0.0).  Fast path (rows of up
// to 65536 candidates): one pass builds a histogram of the top 12 key bits and
// finds the threshold bin; a second pass writes the "strictly above" bitmap
// directly with warp ballots over 32 consecutive candidates and appends the
// keys of the threshold bin to a short list in shared memory; the remaining 20
// key bits are resolved on that list alone (12- and 8-bit digits), and the
// list's winners are OR-ed into the bitmaps.  Every score is read from global
// memory twice at most.  Rows whose threshold bin is too crowded, or longer
// rows, take the general path: the same MSD radix select over every key (rows
// up to 16384 candidates staged in shared memory), bitmaps per 65536-candidate
// segment.  Either way, only when the threshold value is shared by more keys
// than slots left does a scan of the "equal" bitmap pick the lowest indices,
// and one block scan of the bitmap popcounts gives every winner its output
// position, so the list comes out ascending without a sort.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kHistBins = 4096;
constexpr int kSegWords = 2048;              // bitmap segment: 65536 candidates
constexpr int kSegElems = kSegWords * 32;
constexpr int kWordsPerThread = kSegWords / kSelThreads;
constexpr int kCandCap = 8192;               // threshold-bin list of the fast path (max)
constexpr int kStageMax = 16384;             // candidates staged in shared memory (general path, max)
// hist | gtw | eqw | tail: fast path = cand keys + cand idx; general path = staged keys
constexpr int kSelFixedSmem = (kHistBins + 2 * kSegWords) * 4;
constexpr int kSelMaxSmem = kSelFixedSmem + 2 * kCandCap * 4;  // 96 KB: two CTAs per SM
static_assert(kStageMax <= 2 * kCandCap, "staging must fit the tail");

__device__ __forceinline__ uint32_t order_key(float x)
{
    uint32_t b = __float_as_uint(x);
    if ((b << 1) == 0u) b = 0u;  // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SelScratch {
    int warp_tot[kSelWarps];
    int total;
    int digit, above;
    int cand_n;
};

// block-wide exclusive scan of one int per thread; every thread gets the total
__device__ __forceinline__ int block_exclusive_scan(int v, SelScratch *sc, int *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) sc->warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        const int w = lane < kSelWarps ? sc->warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += y;
        }
        if (lane < kSelWarps) sc->warp_tot[lane] = wi - w;  // exclusive prefix of the warps
        if (lane == kSelWarps - 1) sc->total = wi;
    }
    __syncthreads();
    const int res = sc->warp_tot[wid] + incl - v;
    *total = sc->total;
    __syncthreads();
    return res;
}

// Given hist[0 .. nb) of the keys still in play, find the digit whose bin holds
// the need-th largest key.  Returns the digit; *above = keys in higher bins.
__device__ __forceinline__ int find_digit(const uint32_t *hist, int nb, int need, SelScratch *sc, int *above_out)
{
    const int tid = threadIdx.x;
    const int per = nb >= kSelThreads ? nb / kSelThreads : 1;  // digits per thread, highest first
    const int top = nb - tid * per;                             // owns digits [top - per, top)
    int mine = 0;
    if (top > 0)
        for (int q = 1; q <= per; ++q) mine += (int)hist[top - q];
    int tot;
    int above = block_exclusive_scan(mine, sc, &tot);
    if (top > 0) {
        for (int q = 1; q <= per; ++q) {
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

// Ordered emission of one bitmap segment: winners are gtw bits plus, when
// `partial`, the lowest-index eqw bits while the running equal-rank stays below
// `need`; otherwise all eqw bits.  Writes out[pos] = seg0 + bit index.
__device__ __forceinline__ void emit_segment(const uint32_t *gtw, const uint32_t *eqw, int words, int seg0,
                                             bool partial, int need, int need_total, int *out_base,
                                             int *eq_base, int32_t *out, SelScratch *sc)
{
    const int tid = threadIdx.x;
    uint32_t wsel[kWordsPerThread];
    const int w0 = tid * kWordsPerThread;
    if (partial) {
        int ecnt = 0;
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) ecnt += (w0 + q < words) ? __popc(eqw[w0 + q]) : 0;
        int etot;
        int epos = *eq_base + block_exclusive_scan(ecnt, sc, &etot);
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
    int pos = *out_base + block_exclusive_scan(cnt, sc, &stot);
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

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ cu_q,
              const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r,
              int cand_cap, int stage_cap, int32_t *__restrict__ sel)
{
    extern __shared__ uint32_t smem_sel[];
    uint32_t *hist = smem_sel;                     // kHistBins
    uint32_t *gtw = hist + kHistBins;              // kSegWords: key above the threshold
    uint32_t *eqw = gtw + kSegWords;               // kSegWords: key equal to the threshold
    uint32_t *tail = eqw + kSegWords;              // fast path: candidate keys + indices; general: staged keys
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
    if (n <= kSegElems) {
        uint32_t *cand_key = tail;
        uint32_t *cand_idx = tail + cand_cap;
        for (int b = tid; b < kHistBins; b += kSelThreads) hist[b] = 0u;
        for (int w = tid; w < kSegWords; w += kSelThreads) {
            gtw[w] = 0u;
            eqw[w] = 0u;
        }
        if (tid == 0) sc.cand_n = 0;
        __syncthreads();
        // pass 1: histogram of the top 12 key bits (16 keys in flight per thread)
        if ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {
            const float4 *s4 = reinterpret_cast<const float4 *>(srow);
            const int n4 = n >> 2;
            int j = tid;
            for (; j + 3 * kSelThreads < n4; j += 4 * kSelThreads) {
                float4 v[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) v[q] = __ldg(s4 + j + q * kSelThreads);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    atomicAdd(&hist[order_key(v[q].x) >> 20], 1u);
                    atomicAdd(&hist[order_key(v[q].y) >> 20], 1u);
                    atomicAdd(&hist[order_key(v[q].z) >> 20], 1u);
                    atomicAdd(&hist[order_key(v[q].w) >> 20], 1u);
                }
            }
            for (; j < n4; j += kSelThreads) {
                const float4 v = __ldg(s4 + j);
                atomicAdd(&hist[order_key(v.x) >> 20], 1u);
                atomicAdd(&hist[order_key(v.y) >> 20], 1u);
                atomicAdd(&hist[order_key(v.z) >> 20], 1u);
                atomicAdd(&hist[order_key(v.w) >> 20], 1u);
            }
            for (int e = (n4 << 2) + tid; e < n; e += kSelThreads) atomicAdd(&hist[order_key(__ldg(srow + e)) >> 20], 1u);
        } else {
            int j = tid;
            for (; j + 3 * kSelThreads < n; j += 4 * kSelThreads) {
                const float a0 = __ldg(srow + j), a1 = __ldg(srow + j + kSelThreads);
                const float a2 = __ldg(srow + j + 2 * kSelThreads), a3 = __ldg(srow + j + 3 * kSelThreads);
                atomicAdd(&hist[order_key(a0) >> 20], 1u);
                atomicAdd(&hist[order_key(a1) >> 20], 1u);
                atomicAdd(&hist[order_key(a2) >> 20], 1u);
                atomicAdd(&hist[order_key(a3) >> 20], 1u);
            }
            for (; j < n; j += kSelThreads) atomicAdd(&hist[order_key(__ldg(srow + j)) >> 20], 1u);
        }
        __syncthreads();
        int above;
        const int d1 = find_digit(hist, kHistBins, need_total, &sc, &above);
        int need = need_total - above;
        const int cnt1 = (int)hist[d1];
        const uint32_t d1u = (uint32_t)d1;
        if (cnt1 <= cand_cap) {
            // pass 2: bitmap of keys whose top digit is above d1; collect the d1 bin
            const bool take_bin = (need == cnt1);
            const int words = (n + 31) >> 5;
            for (int w0 = wid; w0 < words; w0 += 4 * kSelWarps) {
                uint32_t uu[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // four words' loads in flight
                    const int j = (w0 + q * kSelWarps) * 32 + lane;
                    uu[q] = (w0 + q * kSelWarps < words && j < n) ? order_key(__ldg(srow + j)) : 0u;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int w = w0 + q * kSelWarps;
                    if (w >= words) break;  // uniform across the warp
                    const int j = w * 32 + lane;
                    const bool in = j < n;
                    const uint32_t u = uu[q];
                    const uint32_t dg = u >> 20;
                    const bool gt = in && (dg > d1u || (take_bin && dg == d1u));
                    const bool inbin = in && !take_bin && dg == d1u;
                    const uint32_t gb = __ballot_sync(0xffffffffu, gt);
                    const uint32_t cb = __ballot_sync(0xffffffffu, inbin);
                    int base = 0;
                    if (lane == 0) {
                        gtw[w] = gb;
                        if (cb) base = atomicAdd(&sc.cand_n, __popc(cb));
                    }
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (inbin) {
                        const int p = base + __popc(cb & ((1u << lane) - 1u));
                        cand_key[p] = u;
                        cand_idx[p] = (uint32_t)j;
                    }
                }
            }
            __syncthreads();
            bool partial = false;
            if (!take_bin) {
                const int nc = sc.cand_n;
                // refine the remaining 20 bits on the list: digits 19..8, then 7..0
                uint32_t prefix = d1u << 20, mask = 0xFFF00000u;
                int in_bin = nc;
                const int shifts[2] = {8, 0};
                const int widths[2] = {12, 8};
#pragma unroll 1
                for (int pass = 0; pass < 2; ++pass) {
                    const int nb = 1 << widths[pass];
                    const uint32_t dmask = (uint32_t)nb - 1u;
                    for (int b = tid; b < nb; b += kSelThreads) hist[b] = 0u;
                    __syncthreads();
                    for (int c = tid; c < nc; c += kSelThreads) {
                        const uint32_t u = cand_key[c];
                        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shifts[pass]) & dmask], 1u);
                    }
                    __syncthreads();
                    int ab;
                    const int d = find_digit(hist, nb, need, &sc, &ab);
                    need -= ab;
                    prefix |= (uint32_t)d << shifts[pass];
                    mask |= dmask << shifts[pass];
                    in_bin = (int)hist[d];
                    __syncthreads();
                    if (need == in_bin) break;
                }
                partial = need < in_bin;
                // the list's winners join the bitmaps
                for (int c = tid; c < nc; c += kSelThreads) {
                    const uint32_t u = cand_key[c] & mask;
                    const uint32_t j = cand_idx[c];
                    if (u > prefix) atomicOr(&gtw[j >> 5], 1u << (j & 31));
                    else if (u == prefix) atomicOr(&eqw[j >> 5], 1u << (j & 31));
                }
                __syncthreads();
            }
            emit_segment(gtw, eqw, words, 0, partial, need, need_total, &out_base, &eq_base, out, &sc);
            done = true;
        }
        __syncthreads();
    }

    // ============================ general path ============================
    if (!done) {
        uint32_t *keys = tail;
        const int staged = n < stage_cap ? n : stage_cap;
        for (int j = tid; j < staged; j += kSelThreads) keys[j] = order_key(__ldg(srow + j));
        __syncthreads();
        auto key_at = [&](int j) -> uint32_t { return j < staged ? keys[j] : order_key(__ldg(srow + j)); };
        uint32_t prefix = 0u, mask = 0u;
        int need = need_total, in_bin = 0;
        const int shifts[3] = {20, 8, 0};
        const int widths[3] = {12, 12, 8};
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = shifts[pass];
            const int nb = 1 << widths[pass];
            const uint32_t dmask = (uint32_t)nb - 1u;
            for (int b = tid; b < nb; b += kSelThreads) hist[b] = 0u;
            __syncthreads();
            for (int j = tid; j < n; j += kSelThreads) {
                const uint32_t u = key_at(j);
                if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
            }
            __syncthreads();
            int ab;
            const int d = find_digit(hist, nb, need, &sc, &ab);
            need -= ab;
            prefix |= (uint32_t)d << shift;
            mask |= dmask << shift;
            in_bin = (int)hist[d];
            __syncthreads();
            if (need == in_bin) break;  // the whole threshold bin is taken
        }
        const bool partial = need < in_bin;
        for (int seg0 = 0; seg0 < n; seg0 += kSegElems) {
            const int seg_n = n - seg0 < kSegElems ? n - seg0 : kSegElems;
            const int words = (seg_n + 31) >> 5;
            for (int w = wid; w < words; w += kSelWarps) {
                const int j = seg0 + w * 32 + lane;
                const bool in = j < n;
                const uint32_t u = in ? (key_at(j) & mask) : 0u;
                const uint32_t g = __ballot_sync(0xffffffffu, in && u > prefix);
                const uint32_t e = __ballot_sync(0xffffffffu, in && u == prefix);
                if (lane == 0) {
                    gtw[w] = g;
                    eqw[w] = e;
                }
            }
            __syncthreads();
            emit_segment(gtw, eqw, words, seg0, partial, need, need_total, &out_base, &eq_base, out, &sc);
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
    // shared memory tail: the fast path's candidate list, or the general path's staged keys
    const int cand_cap = (int)(a.ld < kCandCap ? a.ld : kCandCap);
    const int stage_cap = 2 * cand_cap < kStageMax ? 2 * cand_cap : kStageMax;
    const size_t smem = (size_t)kSelFixedSmem + (size_t)2 * cand_cap * sizeof(uint32_t);
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelMaxSmem);
        attr_set = true;
    }
    for (int64_t done = 0; done < rows; done += 0x7FFFFFFF) {
        const int64_t chunk = rows - done < 0x7FFFFFFF ? rows - done : 0x7FFFFFFF;
        select_kernel<<<(unsigned)chunk, kSelThreads, smem, stream>>>(
            a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, cand_cap,
            stage_cap, a.sel);
    }
    return cudaGetLastError();
}

}  // namespace qsa
