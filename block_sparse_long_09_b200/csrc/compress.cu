// compress.cu -- QSA key compressor.
//
// Pooled-key equation ("On the Design of Qwen3.8 Next Architecture", reading
// notes, section 6): kc[b] = RMSNorm(AvgPool(k_idx[b r .. b r + r - 1])).
// Unit gain; eps from the config; QSA_COMPRESS_NO_NORM keeps the plain mean.
//
// HBM-bound: r x 256 B read and 256 B written per block.  One warp per block,
// each lane owns 4 consecutive dims (8-byte loads, 256 B per row per warp:
// fully coalesced).  fp32 arithmetic, bf16 round-to-nearest-even store.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kCompressWarps = 8;

__global__ void __launch_bounds__(kCompressWarps * 32)
compress_kernel(const __nv_bfloat16 *__restrict__ k_idx, const int32_t *__restrict__ cu_k,
                const int32_t *__restrict__ cu_blocks, int batch, int64_t n_items,
                const int32_t *__restrict__ blk_begin, int max_new, int r, int normalise,
                float eps, __nv_bfloat16 *__restrict__ kc)
{
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
        __nv_bfloat162 o0 = __floats2bfloat162_rn(m[0], m[1]);
        __nv_bfloat162 o1 = __floats2bfloat162_rn(m[2], m[3]);
        uint2 packed;
        packed.x = *reinterpret_cast<uint32_t *>(&o0);
        packed.y = *reinterpret_cast<uint32_t *>(&o1);
        *reinterpret_cast<uint2 *>(kc + ((int64_t)cu_blocks[s] + b) * 128 + lane * 4) = packed;
    }
}

}  // namespace

cudaError_t launch_compress(const __nv_bfloat16 *k_idx, const int32_t *cu_k, const int32_t *cu_blocks,
                            int batch, int64_t total_k, const int32_t *blk_begin, int max_new, int r,
                            bool normalise, float eps, __nv_bfloat16 *kc, cudaStream_t stream)
{
    int64_t n_items = blk_begin ? (int64_t)batch * max_new : total_k / r;
    if (n_items <= 0) return cudaSuccess;
    int64_t grid = (n_items + kCompressWarps - 1) / kCompressWarps;
    const int64_t cap = 148 * 16;
    if (grid > cap) grid = cap;
    compress_kernel<<<(unsigned)grid, kCompressWarps * 32, 0, stream>>>(
        k_idx, cu_k, cu_blocks, batch, n_items, blk_begin, max_new, r, normalise ? 1 : 0, eps, kc);
    return cudaGetLastError();
}

}  // namespace qsa
