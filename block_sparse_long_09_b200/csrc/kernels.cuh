// kernels.cuh -- internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <utility>

#include "sm100.cuh"

namespace qsa {

// largest s in [0, batch) with cu[s] <= x (cu ascending prefix sums, cu[0] = 0);
// the last such s, so empty sequences are skipped
__device__ __forceinline__ int find_seq(const int32_t *cu, int batch, int64_t x)
{
    int lo = 0, hi = batch;
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)cu[mid] <= x) lo = mid; else hi = mid;
    }
    return lo;
}

// Indexer scores of one query row against kc blocks [c0, c1) on CUDA cores (the
// decode GEMV, and the fused selector's fallback and rescoring): warp `warp` of
// `nwarps` streams 8 kc rows at a time with 8-byte loads, keeps its 4 heads' slice
// of q in fp32 registers and reduces the 32 (block, head) partial dots with a
// 5-step butterfly reduce-scatter; srow[b] = sum_h w[h] * ReLU(<q[h], kc[b]>).
// kc_at(b) is the address of block b's compressed key (packed or through a page
// table): its hi plane, and 128 values further its lo plane.  kPlanes = 2 adds the
// planes in fp32 before the products (the exact scores); kPlanes = 1 reads the hi
// plane only (half the bytes; each dot then moves by at most |q| |lo|).
template <int kPlanes, typename KcAt>
__device__ __forceinline__ void index_row_cuda_at(const __nv_bfloat16 *__restrict__ q_row,
                                                  const float *__restrict__ w_row, KcAt kc_at, int64_t c0,
                                                  int64_t c1, float *__restrict__ srow, int warp, int nwarps,
                                                  int lane)
{
    float q[4][4];  // this lane's slice of the 4 query heads: dims 4 lane .. 4 lane + 3
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        uint2 raw = *reinterpret_cast<const uint2 *>(q_row + h * 128 + lane * 4);
        float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.x));
        float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.y));
        q[h][0] = a.x; q[h][1] = a.y; q[h][2] = b.x; q[h][3] = b.y;
    }
    const float wv = __ldg(w_row + (lane & 3));
    const int64_t stride = (int64_t)nwarps * 8;
    // the next group's loads are issued before this group's arithmetic: two groups of
    // gathered rows in flight per warp
    uint2 raw[8], rlo[8];
    auto load = [&](int64_t g0, uint2 (&hi)[8], uint2 (&lo)[8]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t b = g0 + j;
            const __nv_bfloat16 *p = b < c1 ? kc_at(b) + lane * 4 : nullptr;
            hi[j] = p != nullptr ? __ldg(reinterpret_cast<const uint2 *>(p)) : make_uint2(0u, 0u);
            if (kPlanes == 2) lo[j] = p != nullptr ? __ldg(reinterpret_cast<const uint2 *>(p + 128)) : make_uint2(0u, 0u);
        }
    };
    if (c0 + warp * 8 < c1) load(c0 + warp * 8, raw, rlo);
    for (int64_t b0 = c0 + warp * 8; b0 < c1; b0 += stride) {
        uint2 nraw[8], nrlo[8];
        if (b0 + stride < c1) load(b0 + stride, nraw, nrlo);
        float v[32];  // v[j * 4 + h] = partial dot of block b0 + j with head h
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw[j].x));
            float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw[j].y));
            if (kPlanes == 2) {
                const float2 al = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&rlo[j].x));
                const float2 bl = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&rlo[j].y));
                a.x += al.x; a.y += al.y; b.x += bl.x; b.y += bl.y;
            }
#pragma unroll
            for (int h = 0; h < 4; ++h)
                v[j * 4 + h] = q[h][0] * a.x + q[h][1] * a.y + q[h][2] * b.x + q[h][3] * b.y;
        }
        // reduce-scatter over the 32 lanes: lane l ends with the full dot of index l
#pragma unroll
        for (int step = 16; step >= 1; step >>= 1) {
            const bool hi = lane & step;
#pragma unroll
            for (int j = 0; j < step; ++j) {
                const float send = hi ? v[j] : v[j + step];
                const float keep = hi ? v[j + step] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, step);
            }
        }
        float sc = wv * fmaxf(v[0], 0.f);  // lane l: block b0 + l/4, head l%4
        sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        sc += __shfl_xor_sync(0xffffffffu, sc, 2);
        const int64_t b = b0 + (lane >> 2);
        if ((lane & 3) == 0 && b < c1) srow[b] = sc;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            raw[j] = nraw[j];
            if (kPlanes == 2) rlo[j] = nrlo[j];
        }
    }
}

// the packed layout: block b of the sequence at kc_seq + 256 b (hi, then lo)
template <int kPlanes = 2>
__device__ __forceinline__ void index_row_cuda(const __nv_bfloat16 *__restrict__ q_row,
                                               const float *__restrict__ w_row, const __nv_bfloat16 *__restrict__ kc_seq,
                                               int64_t c0, int64_t c1, float *__restrict__ srow, int warp,
                                               int nwarps, int lane)
{
    index_row_cuda_at<kPlanes>(q_row, w_row, [=](int64_t b) { return kc_seq + b * 256; }, c0, c1, srow, warp,
                               nwarps, lane);
}

// Partial RoPE of a 128-dim vector held as 4 consecutive dims per lane (lane l: dims
// 4l .. 4l + 3), called by the whole warp: the first rope_dims dims (a multiple of 8)
// rotate in pairs (i, i + rope_dims/2) by pos * base^(-2i / rope_dims), the partner of a
// dim living rope_dims/8 lanes away.  Angle and its sine and cosine in fp64 (positions
// reach 2^18, where an fp32 angle is off by ~1e-2 rad).
struct RopeSpec {
    int dims;    // 0: no rotation
    float base;
};

__device__ __forceinline__ void rope_rotate4(float (&m)[4], int lane, int64_t pos, const RopeSpec &rope)
{
    if (rope.dims <= 0) return;
    const int h = rope.dims / 2;
    const int lo_lanes = h / 4;  // lanes holding dims < h
    const int in_lo = 4 * lane < h, in_hi = !in_lo && 4 * lane < rope.dims;
    const int partner = in_lo ? lane + lo_lanes : (in_hi ? lane - lo_lanes : lane);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float other = __shfl_sync(0xffffffffu, m[c], partner);
        if (in_lo || in_hi) {
            const int i = 4 * lane + c - (in_hi ? h : 0);  // frequency index
            const double a = (double)pos * pow((double)rope.base, -2.0 * (double)i / (double)rope.dims);
            double sn, cs;
            sincos(a, &sn, &cs);
            const float cf = (float)cs, sf = (float)sn;
            // low half: x_i cos - x_{i+h} sin; high half: x_{i} sin + x_{i+h} cos
            m[c] = in_lo ? fmaf(m[c], cf, -other * sf) : fmaf(other, sf, m[c] * cf);
        }
    }
}

cudaError_t launch_rope_queries(const __nv_bfloat16 *q_idx_in, __nv_bfloat16 *q_idx, const int32_t *cu_q,
                                const int32_t *cu_k, int batch, int64_t total_q, int heads, const RopeSpec &rope,
                                cudaStream_t stream);

cudaError_t launch_compress(const __nv_bfloat16 *k_idx, const int32_t *cu_k, const int32_t *cu_blocks,
                            int batch, int64_t total_k, const int32_t *blk_begin, int max_new, int r,
                            bool normalise, float eps, __nv_bfloat16 *kc, cudaStream_t stream,
                            const RopeSpec &rope = RopeSpec{0, 0.f});

struct IndexArgs {
    const __nv_bfloat16 *q_idx;  // [total_q, 4, 128]
    const float *w;              // [total_q, 4]
    const __nv_bfloat16 *kc;     // [kc_rows, 2, 128]: hi plane, then lo plane
    int64_t kc_rows;
    const int32_t *cu_q, *cu_k, *cu_blocks;
    int batch;
    int64_t total_q;
    int64_t row_begin, row_end;
    float *scores;
    int64_t ld;
    int r;
};
cudaError_t launch_index_tc(const IndexArgs &a, cudaStream_t stream);      // tcgen05 GEMM path

// Output of the tcgen05 indexer (index.cu describes the modes): 0 = scores rows,
// 1 = compact sample rows of every stride-th kc tile, 2 = candidate lists.
struct IdxOut {
    int mode;
    float *scores;
    int64_t ld;
    float *sample;
    int64_t sample_ld;
    int stride;
    int64_t min_bt;
    const float *theta;
    uint2 *lists;
    int list_cap;
    int32_t *counts;
};
cudaError_t launch_index_tc_mode(const IndexArgs &a, const IdxOut &out, cudaStream_t stream);
cudaError_t launch_index_rowwise(const IndexArgs &a, cudaStream_t stream); // one-row-per-sequence path
cudaError_t launch_index_rowwise_hi(const IndexArgs &a, cudaStream_t stream);  // the same, hi plane only
// decode rows: the scores into ws, then the selector; refine = hi-plane scan plus the
// exact rescoring of each row's near-threshold window (select.cu)
size_t decode_select_workspace_bytes(int64_t rows, int64_t ld, int grid);
cudaError_t launch_decode_index_select(const IndexArgs &a, int k, void *ws, int grid, bool refine, int32_t *sel,
                                       cudaStream_t stream, int next_n = 1);

struct SelectArgs {
    const float *scores;
    int64_t ld;
    const int32_t *cu_q, *cu_k;
    int batch;
    int64_t row_begin, row_end;
    int32_t *sel;
    int k, r;
    int next_n = 1;  // > 1: decode rows serving next_n queries share one selection (select.cu)
};
cudaError_t launch_select(const SelectArgs &a, cudaStream_t stream);

// A paged decode cache (paged.cu): block_table [batch, max_pages] maps page j of
// sequence s to a page of the pool; a page holds page_size tokens (k_idx rows) and
// page_size / r compressed keys.
struct PagedArgs {
    int64_t num_pages;
    int page_size;
    const int32_t *table;
    int max_pages;
    const int32_t *cu_k;
    int batch, r;
};
cudaError_t launch_compress_paged(const PagedArgs &p, const __nv_bfloat16 *k_pages, __nv_bfloat16 *kc_pages,
                                  const int32_t *blk_begin, int max_new, int64_t max_len_k, bool normalise,
                                  float eps, cudaStream_t stream, const RopeSpec &rope = RopeSpec{0, 0.f});
cudaError_t launch_index_paged(const PagedArgs &p, const __nv_bfloat16 *q_idx, const float *w,
                               const __nv_bfloat16 *kc_pages, float *scores, int64_t ld, cudaStream_t stream);

// Fused prefill index -> select (select.cu): workspace layout and launch.
struct IndexSelectLayout {
    int list_cap, stride;
    int64_t sample_ld, scratch_ld;
    int grid;
    size_t off_sample, off_theta, off_counts, off_lists, off_fb, off_scratch, total;
};
IndexSelectLayout index_select_layout(int64_t rows, int64_t max_len_k, int k, int r, int grid);
size_t index_select_workspace_bytes(int64_t rows, int64_t max_len_k, int k, int r, int grid);
cudaError_t launch_index_select(const IndexArgs &a, int k, void *ws, int grid, int64_t max_len_k, int32_t *sel,
                                cudaStream_t stream);

struct AttnArgs {
    const __nv_bfloat16 *q, *k, *v;  // q [rows_total, 24, 256]; k, v [total_k, 2, 256]
    const int32_t *sel;              // [rows_total, kb]; nullptr = every block (dense)
    const int32_t *cu_q;             // nullptr = decode: row i is sequence i, L_q = 1
    const int32_t *cu_k;
    int batch;
    int64_t total_q, total_k;
    int64_t row_begin, row_end;
    __nv_bfloat16 *o;
    float *lse;
    float *ws;                       // split partials (nsplit > 1), or bounds + partials (chunked)
    int nsplit;
    int kb, r;
    float scale;
    int nchunks = 0;                 // > 1: key-chunked (L2-blocked) schedule
    int chunk_blocks = 0;            // micro-blocks per key chunk
    int even = 0;                    // decode: tiles spread evenly over the CTAs (ws: partial states)
    // decode over a paged K/V cache: k, v are [num_pages * page_size, 2, 256] (total_k rows);
    // block_table [batch, max_pages] maps page j of sequence s to a page of the pool
    const int32_t *block_table = nullptr;
    int page_size = 0, max_pages = 0;
    // decode of a context-parallel shard: the rows attend only selected blocks in
    // [blk_lo[s], blk_hi[s]), whose tokens sit in k, v from row tok_local[s] on (cu_k keeps
    // the sequences' global lengths: positions and causality are global)
    const int64_t *tok_local = nullptr;
    const int32_t *blk_lo = nullptr, *blk_hi = nullptr;
};
cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream);
cudaError_t launch_sparse_decode(const AttnArgs &a, cudaStream_t stream);  // a.even: the decode kernel
// (o, lse) of the same rows from `parts` shards merged by their log-sum-exps
cudaError_t launch_merge_states(const __nv_bfloat16 *o_parts, const float *lse_parts, int parts, int64_t rows,
                                __nv_bfloat16 *o, float *lse, cudaStream_t stream);
// multi-token decode (attn_mtp.cu): next_n <= 4 queries per sequence, one shared selection
int mtp_nsplit(int batch, int kb);
size_t mtp_workspace_bytes(int batch, int kb);
cudaError_t launch_sparse_mtp(const AttnArgs &a, int next_n, cudaStream_t stream);
int dense_decode_nsplit(int64_t max_len_k, int r);  // splits of the dense flash-decoding path
constexpr int kMaxEvenCtas = 256;               // CTAs of the even decode schedule, at most
int even_grid();                                // CTAs of the even decode schedule on this device
size_t even_workspace_bytes(int64_t rows, int grid);  // its partial states (rows + grid slots)
size_t split_workspace_bytes(int64_t rows, int nsplit);  // partial (o, lse) states
size_t chunked_workspace_bytes(int64_t rows, int nchunks);  // bounds + partial states

struct DenseArgs {
    const __nv_bfloat16 *q, *k, *v;
    const int32_t *cu_q, *cu_k;
    int batch;
    int64_t total_q, total_k;
    int max_len_q;
    __nv_bfloat16 *o;
    float *lse;
    float scale;
};
cudaError_t launch_dense_attn(const DenseArgs &a, cudaStream_t stream);

// tensor-map creation (host), defined in api.cu
bool make_tmap_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);
bool make_tmap_2d_f32(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_outer);
bool make_tmap_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2);
int num_sms();
// Launch `kernel` with programmatic stream serialisation: it may be scheduled while the
// previous kernel of the stream still runs, so it must begin with pdl_enter().
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Opt-in dynamic shared memory of `func` on the current device, set once per device
// (thread-safe; later calls on that device only look it up).
cudaError_t set_smem_attr_once(const void *func, int bytes);

}  // namespace qsa
