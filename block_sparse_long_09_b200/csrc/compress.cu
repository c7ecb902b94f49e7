// compress.cu -- QSA key compressor.
//
// Pooled-key equation ("On the Design of Qwen3.8 Next Architecture", reading
// notes, section 6): kc[b] = RMSNorm(AvgPool(k_idx[b r .. b r + r - 1])).
// Unit gain; eps from the config; QSA_COMPRESS_NO_NORM keeps the plain mean.
//
// Output: a compensated bf16 pair per value, kc[b] = hi + lo with hi = bf16(x)
// and lo = bf16(x - hi) (about 16 significant bits).  A plain bf16 kc moves the
// indexer scores by up to a few percent where a dot product is small against
// the vectors' norms, which changes top-k selections; the pair keeps the
// scores within ~1e-5 of the fp32 value while the indexer still runs bf16
// tensor-core MMAs (one per plane).
//
// HBM-bound: r x 256 B read and 512 B written per block.  One warp per block,
// each lane owns 4 consecutive dims (8-byte loads, 256 B per row per warp:
// fully coalesced).  fp32 arithmetic, round-to-nearest-even stores.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kCompressWarps = 8;

__global__ void __launch_bounds__(kCompressWarps * 32)
compress_kernel(const __nv_bfloat16 *__restrict__ k_idx, const int32_t *__restrict__ cu_k,
                const int32_t *__restrict__ cu_blocks, int batch, int64_t n_items,
                const int32_t *__restrict__ blk_begin, int max_new, int r, int normalise,
                float eps, __nv_bfloat16 *__restrict__ kc, const RopeSpec rope)
{
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = (int64_t)blockIdx.x * kCompressWarps + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kCompressWarps;
    const int64_t total_blocks = cu_blocks[batch];

    for (int64_t item = warp_global; item < n_items; item += nwarps) {
        int s;
        int64_t b;
        if (blk_begin == nullptr) {
            if (item >= total_blocks) break;
            s = find_seq(cu_blocks, batch, item);
            b = item - cu_blocks[s];
        } else {
            s = (int)(item / max_new);
            int32_t b0 = blk_begin[s];
            if (b0 < 0) {
                if (lane == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
                continue;
            }
            b = (int64_t)b0 + item % max_new;
        }
        const int64_t Lk = (int64_t)cu_k[s + 1] - cu_k[s];
        const int64_t nb = (int64_t)cu_blocks[s + 1] - cu_blocks[s];
        if (nb != Lk / r) {
            if (lane == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
            continue;
        }
        if (b >= nb) continue;

        const __nv_bfloat16 *src = k_idx + ((int64_t)cu_k[s] + b * r) * 128 + lane * 4;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < r; ++j) {
            uint2 raw = *reinterpret_cast<const uint2 *>(src + (int64_t)j * 128);
            __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
            __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
            float2 flo = __bfloat1622float2(lo), fhi = __bfloat1622float2(hi);
            acc[0] += flo.x; acc[1] += flo.y; acc[2] += fhi.x; acc[3] += fhi.y;
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
        __nv_bfloat162 h0 = __floats2bfloat162_rn(m[0], m[1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(m[2], m[3]);
        const float2 fh0 = __bfloat1622float2(h0), fh1 = __bfloat1622float2(h1);
        __nv_bfloat162 l0 = __floats2bfloat162_rn(m[0] - fh0.x, m[1] - fh0.y);
        __nv_bfloat162 l1 = __floats2bfloat162_rn(m[2] - fh1.x, m[3] - fh1.y);
        uint2 hi, lo;
        hi.x = *reinterpret_cast<uint32_t *>(&h0);
        hi.y = *reinterpret_cast<uint32_t *>(&h1);
        lo.x = *reinterpret_cast<uint32_t *>(&l0);
        lo.y = *reinterpret_cast<uint32_t *>(&l1);
        __nv_bfloat16 *dst = kc + ((int64_t)cu_blocks[s] + b) * 256 + lane * 4;
        *reinterpret_cast<uint2 *>(dst) = hi;
        *reinterpret_cast<uint2 *>(dst + 128) = lo;
    }
}

// partial RoPE of indexer query rows: one warp per (row, head), 4 dims per lane
constexpr int kRopeWarps = 8;

__global__ void __launch_bounds__(kRopeWarps * 32)
rope_queries_kernel(const __nv_bfloat16 *__restrict__ q_in, __nv_bfloat16 *__restrict__ q_out,
                    const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k, int batch,
                    int64_t total_q, int heads, const RopeSpec rope)
{
    const int lane = threadIdx.x & 31;
    const int64_t n_items = total_q * heads;
    for (int64_t item = (int64_t)blockIdx.x * kRopeWarps + (threadIdx.x >> 5); item < n_items;
         item += (int64_t)gridDim.x * kRopeWarps) {
        const int64_t i = item / heads;
        const int s = find_seq(cu_q, batch, i);
        const int64_t Lq = (int64_t)cu_q[s + 1] - cu_q[s], Lk = (int64_t)cu_k[s + 1] - cu_k[s];
        const int64_t t = (Lk - Lq) + (i - cu_q[s]);
        const int64_t off = item * 128 + lane * 4;
        const uint2 raw = *reinterpret_cast<const uint2 *>(q_in + off);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
        const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
        float m[4] = {a.x, a.y, c.x, c.y};
        rope_rotate4(m, lane, t, rope);
        __nv_bfloat162 o0 = __floats2bfloat162_rn(m[0], m[1]), o1 = __floats2bfloat162_rn(m[2], m[3]);
        uint2 w;
        w.x = *reinterpret_cast<uint32_t *>(&o0);
        w.y = *reinterpret_cast<uint32_t *>(&o1);
        *reinterpret_cast<uint2 *>(q_out + off) = w;
    }
}

}  // namespace

cudaError_t launch_rope_queries(const __nv_bfloat16 *q_idx_in, __nv_bfloat16 *q_idx, const int32_t *cu_q,
                                const int32_t *cu_k, int batch, int64_t total_q, int heads, const RopeSpec &rope,
                                cudaStream_t stream)
{
    const int64_t n_items = total_q * heads;
    if (n_items <= 0) return cudaSuccess;
    int64_t grid = (n_items + kRopeWarps - 1) / kRopeWarps;
    if (grid > 148 * 16) grid = 148 * 16;
    rope_queries_kernel<<<(unsigned)grid, kRopeWarps * 32, 0, stream>>>(q_idx_in, q_idx, cu_q, cu_k, batch,
                                                                        total_q, heads, rope);
    return cudaGetLastError();
}

cudaError_t launch_compress(const __nv_bfloat16 *k_idx, const int32_t *cu_k, const int32_t *cu_blocks,
                            int batch, int64_t total_k, const int32_t *blk_begin, int max_new, int r,
                            bool normalise, float eps, __nv_bfloat16 *kc, cudaStream_t stream,
                            const RopeSpec &rope)
{
    int64_t n_items = blk_begin ? (int64_t)batch * max_new : total_k / r;
    if (n_items <= 0) return cudaSuccess;
    int64_t grid = (n_items + kCompressWarps - 1) / kCompressWarps;
    const int64_t cap = 148 * 16;
    if (grid > cap) grid = cap;
    return launch_pdl(compress_kernel, dim3((unsigned)grid), dim3(kCompressWarps * 32), 0, stream, k_idx, cu_k,
                      cu_blocks, batch, n_items, blk_begin, max_new, r, normalise ? 1 : 0, eps, kc, rope);
}

}  // namespace qsa
