// paged.cu -- the compressed-key side of a paged decode cache: the compressor and
// the one-row indexer reading and writing through a block table.
//
// A paged serving cache keeps every per-token tensor of a sequence in fixed-size
// pages found through one block table ("结果 2" of the reading notes of "On the
// Design of Qwen3.8 Next Architecture": the dense baseline is a paged GQA
// cache).  Page p holds page_size tokens: K and V rows (read by the paged decode
// attention), the raw indexer keys k_idx [page_size, 128] bf16, and their
// compressed keys kc [page_size / r, 2, 128] bf16 hi/lo pairs (section 6, pooled-key
// equation).  page_size is a multiple of r, so a micro-block never straddles a
// page, and block b of a sequence lives in page table[b r / page_size] at
// compressed row (b r % page_size) / r.
//
// The arithmetic is the packed path's: the compressor is the same warp-per-block
// RMSNorm of the block mean (compensated bf16 pair), the indexer the same CUDA-core GEMV
// (index_row_cuda_at) with the page translation in the block address.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kPagedWarps = 8;
constexpr int kPagedChunk = 1024;  // kc blocks per CTA of the indexer

// page row of token position tok of sequence s, or -1 (flagged) when the table has none
__device__ __forceinline__ int64_t page_row(const int32_t *table, int max_pages, int64_t num_pages, int page_size,
                                            int64_t s, int64_t tok)
{
    const int64_t j = tok / page_size;
    const int32_t page = j < max_pages ? __ldg(table + s * max_pages + j) : -1;
    if (page < 0 || page >= num_pages) return -1;
    return (int64_t)page * page_size + tok % page_size;
}

__global__ void __launch_bounds__(kPagedWarps * 32)
compress_paged_kernel(const __nv_bfloat16 *__restrict__ k_pages, __nv_bfloat16 *__restrict__ kc_pages, int64_t num_pages,
                      int page_size, const int32_t *__restrict__ table, int max_pages,
                      const int32_t *__restrict__ cu_k, int batch, const int32_t *__restrict__ blk_begin,
                      int max_new, int64_t blocks_per_seq, int r, int normalise, float eps, const RopeSpec rope)
{
    const int lane = threadIdx.x & 31;
    const int64_t n_items = (int64_t)batch * (blk_begin != nullptr ? max_new : blocks_per_seq);
    const int64_t per = blk_begin != nullptr ? max_new : blocks_per_seq;
    for (int64_t item = (int64_t)blockIdx.x * kPagedWarps + (threadIdx.x >> 5); item < n_items;
         item += (int64_t)gridDim.x * kPagedWarps) {
        const int s = (int)(item / per);
        int64_t b = item % per;
        if (blk_begin != nullptr) {
            const int32_t b0 = __ldg(blk_begin + s);
            if (b0 < 0) {
                if (lane == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
                continue;
            }
            b += b0;
        }
        const int64_t Lk = (int64_t)__ldg(cu_k + s + 1) - __ldg(cu_k + s);
        if (b >= Lk / r) continue;  // incomplete (or absent) block
        const int64_t row = page_row(table, max_pages, num_pages, page_size, s, b * r);
        if (row < 0) {
            if (lane == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
            continue;
        }
        const __nv_bfloat16 *src = k_pages + row * 128 + lane * 4;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < r; ++j) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(src + (int64_t)j * 128);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
            const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
            acc[0] += a.x; acc[1] += a.y; acc[2] += c.x; acc[3] += c.y;
        }
        const float inv_r = 1.0f / (float)r;
        float m[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) m[c] = acc[c] * inv_r;
        if (normalise) {
            float ss = m[0] * m[0] + m[1] * m[1] + m[2] * m[2] + m[3] * m[3];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv = rsqrtf(ss * (1.0f / 128.0f) + eps);
#pragma unroll
            for (int c = 0; c < 4; ++c) m[c] *= inv;
        }
        rope_rotate4(m, lane, b * r, rope);  // the pooled key at its block's first position
        // the compensated pair: hi = bf16(x), lo = bf16(x - hi)
        const __nv_bfloat162 h0 = __floats2bfloat162_rn(m[0], m[1]);
        const __nv_bfloat162 h1 = __floats2bfloat162_rn(m[2], m[3]);
        const float2 fh0 = __bfloat1622float2(h0), fh1 = __bfloat1622float2(h1);
        const __nv_bfloat162 l0 = __floats2bfloat162_rn(m[0] - fh0.x, m[1] - fh0.y);
        const __nv_bfloat162 l1 = __floats2bfloat162_rn(m[2] - fh1.x, m[3] - fh1.y);
        uint2 hi, lo;
        hi.x = *reinterpret_cast<const uint32_t *>(&h0);
        hi.y = *reinterpret_cast<const uint32_t *>(&h1);
        lo.x = *reinterpret_cast<const uint32_t *>(&l0);
        lo.y = *reinterpret_cast<const uint32_t *>(&l1);
        __nv_bfloat16 *dst = kc_pages + (row / r) * 256 + lane * 4;
        *reinterpret_cast<uint2 *>(dst) = hi;
        *reinterpret_cast<uint2 *>(dst + 128) = lo;
    }
}

// one query per sequence (t = L - 1): scores of blocks [c0, c1) of its b_t candidates
__global__ void __launch_bounds__(kPagedWarps * 32)
index_paged_kernel(const __nv_bfloat16 *__restrict__ q_idx, const float *__restrict__ w,
                   const __nv_bfloat16 *__restrict__ kc_pages, int64_t num_pages, int page_size,
                   const int32_t *__restrict__ table, int max_pages, const int32_t *__restrict__ cu_k, int r,
                   float *__restrict__ scores, int64_t ld)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t s = blockIdx.y;
    const int64_t t = (int64_t)__ldg(cu_k + s + 1) - __ldg(cu_k + s) - 1;
    int64_t bt = t >= 0 ? t / r : 0;
    if (bt > ld) {
        if (threadIdx.x == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        bt = ld;
    }
    const int64_t c0 = (int64_t)blockIdx.x * kPagedChunk;
    const int64_t c1 = c0 + kPagedChunk < bt ? c0 + kPagedChunk : bt;
    if (c0 >= c1) return;
    const int bpp = page_size / r;  // compressed rows per page
    auto kc_at = [=](int64_t b) -> const __nv_bfloat16 * {
        const int64_t j = b / bpp;
        const int32_t page = j < max_pages ? __ldg(table + s * max_pages + j) : -1;
        if (page < 0 || page >= num_pages) {  // reads row 0 instead, and flags
            set_device_status(QSA_ERR_DEVICE_CHECK);
            return kc_pages;
        }
        return kc_pages + ((int64_t)page * bpp + b % bpp) * 256;
    };
    index_row_cuda_at<2>(q_idx + s * 512, w + s * 4, kc_at, c0, c1, scores + s * ld, warp, kPagedWarps, lane);
}

}  // namespace

cudaError_t launch_compress_paged(const PagedArgs &p, const __nv_bfloat16 *k_pages, __nv_bfloat16 *kc_pages,
                                  const int32_t *blk_begin, int max_new, int64_t max_len_k, bool normalise,
                                  float eps, cudaStream_t stream, const RopeSpec &rope)
{
    const int64_t per = blk_begin != nullptr ? max_new : max_len_k / p.r;
    const int64_t n_items = (int64_t)p.batch * per;
    if (n_items <= 0) return cudaSuccess;
    int64_t grid = (n_items + kPagedWarps - 1) / kPagedWarps;
    if (grid > 148 * 16) grid = 148 * 16;
    compress_paged_kernel<<<(unsigned)grid, kPagedWarps * 32, 0, stream>>>(
        k_pages, kc_pages, p.num_pages, p.page_size, p.table, p.max_pages, p.cu_k, p.batch, blk_begin, max_new,
        max_len_k / p.r, p.r, normalise ? 1 : 0, eps, rope);
    return cudaGetLastError();
}

cudaError_t launch_index_paged(const PagedArgs &p, const __nv_bfloat16 *q_idx, const float *w,
                               const __nv_bfloat16 *kc_pages, float *scores, int64_t ld, cudaStream_t stream)
{
    if (p.batch <= 0) return cudaSuccess;
    const int64_t chunks = (ld + kPagedChunk - 1) / kPagedChunk;
    if (p.batch > 65535 || chunks <= 0) return cudaErrorInvalidValue;
    index_paged_kernel<<<dim3((unsigned)chunks, (unsigned)p.batch), kPagedWarps * 32, 0, stream>>>(
        q_idx, w, kc_pages, p.num_pages, p.page_size, p.table, p.max_pages, p.cu_k, p.r, scores, ld);
    return cudaGetLastError();
}

}  // namespace qsa
