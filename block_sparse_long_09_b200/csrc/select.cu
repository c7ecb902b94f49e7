// select.cu -- QSA top-k micro-block selection.
//
// Budget sentence of "On the Design of Qwen3.8 Next Architecture" (reading
// notes, section 6): per query, the own (trailing, possibly incomplete) causal
// block b_t is always kept and the remaining k - 1 slots go to the best complete
// blocks 0 .. b_t - 1.  Ties go to the lower block index; the output lists the
// chosen blocks in ascending order, padded with -1.
//
// One CTA (512 threads) per query row.  The fp32 scores become order-preserving
// 32-bit keys (sign-flip trick, -0.0 folded into +0.0); rows up to 32768
// candidates are staged once in shared memory, longer rows keep their tail in
// global memory (L2).  The (k-1)-th largest key is found by an MSD radix select
// with 12-, 12- and 8-bit digits (one shared histogram, a block-wide suffix scan
// per digit), stopping as soon as the whole threshold bin is taken.  The winners
// are then marked in bitmaps built with warp ballots over 32 consecutive
// candidates -- "above the threshold" and "equal to it" -- and only when the
// threshold value is shared by more keys than slots left does a scan of the
// "equal" bitmap pick the lowest indices.  One block scan of the bitmap
// popcounts gives every winner its output position, so the list comes out
// ascending without a sort.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kHistBins = 4096;
constexpr int kSegWords = 2048;              // bitmap segment: 65536 candidates
constexpr int kWordsPerThread = kSegWords / kSelThreads;
constexpr int kStageMax = 32768;             // candidates staged in shared memory
constexpr int kSelFixedSmem = (kHistBins + 2 * kSegWords) * 4;

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

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ cu_q,
              const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r,
              int stage_cap, int32_t *__restrict__ sel)
{
    extern __shared__ uint32_t smem_sel[];
    uint32_t *hist = smem_sel;                     // kHistBins
    uint32_t *gtw = hist + kHistBins;              // kSegWords: key above the threshold
    uint32_t *eqw = gtw + kSegWords;               // kSegWords: key equal to the threshold
    uint32_t *keys = eqw + kSegWords;              // staged keys
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
    const int staged = n < stage_cap ? n : stage_cap;
    if (((reinterpret_cast<uintptr_t>(srow)) & 15u) == 0) {
        const int n4 = staged >> 2;
        for (int j = tid; j < n4; j += kSelThreads) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(srow) + j);
            reinterpret_cast<uint4 *>(keys)[j] = make_uint4(order_key(v.x), order_key(v.y), order_key(v.z), order_key(v.w));
        }
        for (int j = (n4 << 2) + tid; j < staged; j += kSelThreads) keys[j] = order_key(__ldg(srow + j));
    } else {
        for (int j = tid; j < staged; j += kSelThreads) keys[j] = order_key(__ldg(srow + j));
    }
    __syncthreads();
    auto key_at = [&](int j) -> uint32_t { return j < staged ? keys[j] : order_key(__ldg(srow + j)); };

    // ---------------- radix select of the (k-1)-th largest key ----------------
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
        // thread owns `per` consecutive digits, highest digits first
        const int per = nb >= kSelThreads ? nb / kSelThreads : 1;
        const int top = nb - tid * per;          // owns digits [top - per, top)
        int mine = 0;
        if (top > 0)
            for (int q = 1; q <= per; ++q) mine += (int)hist[top - q];
        int tot;
        int above = block_exclusive_scan(mine, &sc, &tot);
        if (top > 0) {
            for (int q = 1; q <= per; ++q) {
                const int h = (int)hist[top - q];
                if (above < need && above + h >= need) {
                    sc.digit = top - q;
                    sc.above = above;
                }
                above += h;
            }
        }
        __syncthreads();
        const int digit = sc.digit;
        need -= sc.above;
        prefix |= (uint32_t)digit << shift;
        mask |= dmask << shift;
        in_bin = (int)hist[digit];
        __syncthreads();
        if (need == in_bin) break;  // the whole threshold bin is taken
    }
    const bool partial = need < in_bin;  // only some keys equal to the threshold are taken

    // ---------------- ordered emission through bitmaps ----------------
    int out_base = 0, eq_base = 0;
    for (int seg0 = 0; seg0 < n; seg0 += kSegWords * 32) {
        const int seg_n = n - seg0 < kSegWords * 32 ? n - seg0 : kSegWords * 32;
        const int words = (seg_n + 31) >> 5;
        for (int w = wid; w < words; w += kSelWarps) {
            const int j = seg0 + w * 32 + lane;
            uint32_t u = 0u;
            const bool in = j < n;
            if (in) u = key_at(j) & mask;
            const uint32_t g = __ballot_sync(0xffffffffu, in && u > prefix);
            const uint32_t e = __ballot_sync(0xffffffffu, in && u == prefix);
            if (lane == 0) {
                gtw[w] = g;
                eqw[w] = e;
            }
        }
        __syncthreads();
        uint32_t wsel[kWordsPerThread];
        const int w0 = tid * kWordsPerThread;
        if (partial) {
            int ecnt = 0;
#pragma unroll
            for (int q = 0; q < kWordsPerThread; ++q) ecnt += (w0 + q < words) ? __popc(eqw[w0 + q]) : 0;
            int etot;
            int epos = eq_base + block_exclusive_scan(ecnt, &sc, &etot);
#pragma unroll
            for (int q = 0; q < kWordsPerThread; ++q) {
                uint32_t e = (w0 + q < words) ? eqw[w0 + q] : 0u;
                // keep the lowest set bits while the running rank stays below `need`
                uint32_t taken = 0u;
                while (e != 0u && epos < need) {
                    const uint32_t lowbit = e & (~e + 1u);
                    taken |= lowbit;
                    e ^= lowbit;
                    ++epos;
                }
                epos += __popc(e);
                wsel[q] = ((w0 + q < words) ? gtw[w0 + q] : 0u) | taken;
            }
            eq_base += etot;
        } else {
#pragma unroll
            for (int q = 0; q < kWordsPerThread; ++q) wsel[q] = (w0 + q < words) ? (gtw[w0 + q] | eqw[w0 + q]) : 0u;
        }
        int cnt = 0;
#pragma unroll
        for (int q = 0; q < kWordsPerThread; ++q) cnt += __popc(wsel[q]);
        int stot;
        int pos = out_base + block_exclusive_scan(cnt, &sc, &stot);
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
        out_base += stot;
        __syncthreads();
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
    const int64_t cap = a.ld < kStageMax ? a.ld : kStageMax;
    const size_t smem = (size_t)kSelFixedSmem + (size_t)cap * sizeof(uint32_t);
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSelFixedSmem + kStageMax * (int)sizeof(uint32_t));
        attr_set = true;
    }
    for (int64_t done = 0; done < rows; done += 0x7FFFFFFF) {
        const int64_t chunk = rows - done < 0x7FFFFFFF ? rows - done : 0x7FFFFFFF;
        select_kernel<<<(unsigned)chunk, kSelThreads, smem, stream>>>(
            a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r, (int)cap, a.sel);
    }
    return cudaGetLastError();
}

}  // namespace qsa
