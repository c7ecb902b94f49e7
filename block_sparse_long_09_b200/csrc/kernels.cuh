// kernels.cuh -- internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

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

cudaError_t launch_compress(const __nv_bfloat16 *k_idx, const int32_t *cu_k, const int32_t *cu_blocks,
                            int batch, int64_t total_k, const int32_t *blk_begin, int max_new, int r,
                            bool normalise, float eps, __nv_bfloat16 *kc, cudaStream_t stream);

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
cudaError_t launch_index_rowwise(const IndexArgs &a, cudaStream_t stream); // one-row-per-sequence path

struct SelectArgs {
    const float *scores;
    int64_t ld;
    const int32_t *cu_q, *cu_k;
    int batch;
    int64_t row_begin, row_end;
    int32_t *sel;
    int k, r;
};
cudaError_t launch_select(const SelectArgs &a, cudaStream_t stream);

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
};
cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream);
cudaError_t launch_sparse_decode(const AttnArgs &a, cudaStream_t stream);  // a.even: the decode kernel
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
// Opt-in dynamic shared memory of `func` on the current device, set once per device
// (thread-safe; later calls on that device only look it up).
cudaError_t set_smem_attr_once(const void *func, int bytes);

}  // namespace qsa
