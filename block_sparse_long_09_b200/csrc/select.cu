// select.cu -- QSA top-k micro-block selection.
//
// Budget sentence of "On the Design of Qwen3.8 Next Architecture" (reading
// notes, section 6): per query, the own (trailing, possibly incomplete) causal
// block b_t is always kept and the remaining k - 1 slots go to the best complete
// blocks 0 .. b_t - 1.  Ties go to the lower block index; the output lists the
// chosen blocks in ascending order, padded with -1.
//
// One CTA per query row.  The fp32 scores are mapped to an order-preserving
// 32-bit key (sign-flip trick, -0.0 folded into +0.0) and the (k-1)-th largest
// key is found by an MSD radix select (8-bit digits, privatised per-warp
// histograms, stop early once the whole threshold bin is taken).  A final pass
// compacts the winners in index order, so "equal to the threshold" keys are
// taken lowest-index-first exactly as the tie rule asks, and the output comes
// out ascending without a sort.  Rows that fit are staged once in shared
// memory; longer rows are re-read from global memory (L2) on each pass.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelSmemKeys = 32768;  // rows up to this many candidates are staged in smem

__device__ __forceinline__ uint32_t order_key(float x)
{
    uint32_t b = __float_as_uint(x);
    if ((b << 1) == 0u) b = 0u;  // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// block-wide exclusive scan of a 0/1 flag in index order; returns this thread's
// exclusive prefix, *total = number of set flags in the block
__device__ __forceinline__ int block_scan_flag(bool flag, int *warp_tot, int *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[wid] = __popc(ballot);
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
        int c = warp_tot[w];
        before += (w < wid) ? c : 0;
        tot += c;
    }
    __syncthreads();
    *total = tot;
    return before + in_warp;
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ cu_q,
              const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int k, int r,
              int smem_keys, int32_t *__restrict__ sel)
{
    extern __shared__ uint32_t keys_smem[];
    __shared__ int whist[kSelWarps][256];
    __shared__ int hist[256];
    __shared__ int warp_tot[kSelWarps];
    __shared__ int s_digit, s_above;

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
    if (bt > ld) {  // scores row too short for this query
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
    const bool staged = n <= smem_keys;
    if (staged) {
        for (int j = tid; j < n; j += kSelThreads) keys_smem[j] = order_key(srow[j]);
        __syncthreads();
    }
    auto key_at = [&](int j) -> uint32_t { return staged ? keys_smem[j] : order_key(__ldg(srow + j)); };

    uint32_t prefix = 0u, mask = 0u;
    int need = need_total;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int j = tid; j < kSelWarps * 256; j += kSelThreads) (&whist[0][0])[j] = 0;
        __syncthreads();
        for (int j = tid; j < n; j += kSelThreads) {
            const uint32_t u = key_at(j);
            if ((u & mask) == prefix) atomicAdd(&whist[wid][(u >> shift) & 255u], 1);
        }
        __syncthreads();
        if (tid < 256) {
            int c = 0;
#pragma unroll
            for (int w = 0; w < kSelWarps; ++w) c += whist[w][tid];
            hist[tid] = c;
        }
        __syncthreads();
        // suffix sums over digits 255 .. 0: warp 0 scans 8 digits per lane
        if (wid == 0) {
            int local[8], sum = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {  // lane owns digits 255 - 8 lane - q
                local[q] = hist[255 - 8 * lane - q];
                sum += local[q];
            }
            int incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            int above = incl - sum;  // count of keys in digits above this lane's range
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (above < need && above + local[q] >= need) {
                    s_digit = 255 - 8 * lane - q;
                    s_above = above;
                }
                above += local[q];
            }
        }
        __syncthreads();
        const int digit = s_digit;
        need -= s_above;
        prefix |= (uint32_t)digit << shift;
        mask |= 0xFFu << shift;
        const int in_bin = hist[digit];
        __syncthreads();
        if (need == in_bin) break;  // the whole threshold bin is taken: no tie left to break
    }

    // ordered compaction: keys above the threshold prefix, plus the first `need`
    // keys equal to it (lowest block indices first)
    int written = 0, eq_seen = 0;
    for (int base = 0; base < n; base += kSelThreads) {
        const int j = base + tid;
        uint32_t u = 0u;
        if (j < n) u = key_at(j) & mask;
        const bool gt = j < n && u > prefix;
        const bool eq = j < n && u == prefix;
        int eq_tot;
        const int eq_rank = eq_seen + block_scan_flag(eq, warp_tot, &eq_tot);
        const bool take = gt || (eq && eq_rank < need);
        int take_tot;
        const int pos = written + block_scan_flag(take, warp_tot, &take_tot);
        if (take && pos < need_total) out[pos] = j;
        written += take_tot;
        eq_seen += eq_tot;
    }
    if (tid == 0) {
        if (written != need_total) set_device_status(QSA_ERR_DEVICE_CHECK);
        out[need_total] = (int32_t)bt;
    }
    (void)lane;
}

}  // namespace

cudaError_t launch_select(const SelectArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0) return cudaSuccess;
    int64_t keys = a.ld < kSelSmemKeys ? a.ld : kSelSmemKeys;
    size_t smem = (size_t)keys * sizeof(uint32_t);
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSelSmemKeys * (int)sizeof(uint32_t));
        attr_set = true;
    }
    for (int64_t done = 0; done < rows; done += 0x7FFFFFFF) {
        int64_t chunk = rows - done < 0x7FFFFFFF ? rows - done : 0x7FFFFFFF;
        select_kernel<<<(unsigned)chunk, kSelThreads, smem, stream>>>(
            a.scores + done * a.ld, a.ld, a.cu_q, a.cu_k, a.batch, a.row_begin + done, a.k, a.r,
            (int)keys, a.sel);
    }
    return cudaGetLastError();
}

}  // namespace qsa
