// api.cu -- the extern "C" entry points of libqsa.so (declared in include/qsa.h):
// host-side argument validation, tensor-map creation and kernel dispatch.
// Nothing here allocates device memory; every buffer is the caller's.
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"

namespace qsa {

__device__ int g_device_status = 0;
#ifdef QSA_DEBUG_CHECKS
__device__ int g_debug_fault_site = 0;
#endif

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// one NVTX range per entry point, named after it (a no-op unless a profiler is attached)
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

}  // namespace

bool make_tmap_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                  uint32_t box_inner, uint32_t box_outer)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr || !aligned16(base) || (row_bytes & 15u) != 0 || outer == 0) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_2d_f32(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                      uint32_t box_inner, uint32_t box_outer)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr || !aligned16(base) || (row_bytes & 15u) != 0 || outer == 0 || inner == 0) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr || !aligned16(base) || (stride1_bytes & 15u) != 0 || (stride2_bytes & 15u) != 0 || d2 == 0)
        return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t set_smem_attr_once(const void *func, int bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    struct Done {
        const void *func;
        int dev, bytes;
    };
    static std::mutex mu;
    static std::vector<Done> done;
    std::lock_guard<std::mutex> lock(mu);
    for (const Done &d : done)
        if (d.func == func && d.dev == dev && d.bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.push_back(Done{func, dev, bytes});
    return e;
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

}  // namespace qsa

using namespace qsa;

namespace {

qsa_status check_config(const qsa_config *c)
{
    if (c == nullptr) return QSA_ERR_INVALID_ARG;
    if (c->r <= 0 || c->budget_blocks <= 0 || c->n_heads_q <= 0 || c->n_heads_kv <= 0 || c->head_dim <= 0 ||
        c->n_heads_idx <= 0 || c->idx_dim <= 0 || !(c->softmax_scale > 0.f) || !(c->rms_eps >= 0.f) ||
        c->kv_chunk_blocks < 0)
        return QSA_ERR_INVALID_ARG;
    if (c->r != 4 || c->budget_blocks > 2048 || c->n_heads_q != 24 || c->n_heads_kv != 2 || c->head_dim != 256 ||
        c->n_heads_idx != 4 || c->idx_dim != 128 || (c->flags & ~(QSA_COMPRESS_NO_NORM | QSA_INDEX_ROPE)) != 0)
        return QSA_ERR_UNSUPPORTED;
    if ((c->flags & QSA_INDEX_ROPE) != 0 &&
        (c->rope_dims < 8 || c->rope_dims > c->idx_dim || c->rope_dims % 8 != 0 || !(c->rope_base > 1.f) ||
         !(c->rope_base < 3.0e38f)))
        return QSA_ERR_INVALID_ARG;
    return QSA_OK;
}

// the pooled keys' partial RoPE of a config (dims 0: none)
qsa::RopeSpec rope_of(const qsa_config *c)
{
    return (c->flags & QSA_INDEX_ROPE) != 0 ? qsa::RopeSpec{c->rope_dims, c->rope_base} : qsa::RopeSpec{0, 0.f};
}

qsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }

// key-chunked (L2-blocked) prefill schedule: opt-in through cfg->kv_chunk_blocks > 0
int nchunks_of(const qsa_config *c, int64_t max_len_k)
{
    if (c->kv_chunk_blocks <= 0) return 1;
    const int64_t blocks = (max_len_k + c->r - 1) / c->r;
    const int64_t cb = c->kv_chunk_blocks;
    const int64_t n = (blocks + cb - 1) / cb;
    return (int)(n > 0 ? (n < 4096 ? n : 4096) : 1);
}

const __nv_bfloat16 *bf(const qsa_bf16 *p) { return reinterpret_cast<const __nv_bfloat16 *>(p); }
__nv_bfloat16 *bf(qsa_bf16 *p) { return reinterpret_cast<__nv_bfloat16 *>(p); }
bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

void qsa_config_init(qsa_config *cfg)
{
    if (cfg == nullptr) return;
    cfg->r = 4;
    cfg->budget_blocks = 512;
    cfg->n_heads_q = 24;
    cfg->n_heads_kv = 2;
    cfg->head_dim = 256;
    cfg->n_heads_idx = 4;
    cfg->idx_dim = 128;
    cfg->softmax_scale = 0.0625f;
    cfg->rms_eps = 1e-6f;
    cfg->flags = 0u;
    cfg->kv_chunk_blocks = 0;
    cfg->rope_dims = 64;
    cfg->rope_base = 10000.f;
}

int32_t qsa_version(void) { return 100; }

const char *qsa_status_string(qsa_status s)
{
    switch (s) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG: a pointer, size or range argument is invalid";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED: configuration outside the supported model shape";
    case QSA_ERR_WORKSPACE_TOO_SMALL: return "QSA_ERR_WORKSPACE_TOO_SMALL: workspace smaller than qsa_workspace_size()";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA: a CUDA launch or runtime call failed";
    case QSA_ERR_TIMEOUT: return "QSA_ERR_TIMEOUT: a bounded device-side wait gave up";
    case QSA_ERR_DEVICE_CHECK: return "QSA_ERR_DEVICE_CHECK: a kernel found an out-of-range index and skipped it";
    case QSA_ERR_SCRATCH_LIMIT:
        return "QSA_ERR_SCRATCH_LIMIT: the call needs more than the library's fixed 16 MiB decode scratch "
               "(QSA_STATIC_SCRATCH_BYTES); use qsa_sparse_attn_decode with a workspace";
    default: return "QSA: unknown status";
    }
}

size_t qsa_workspace_size(const qsa_config *cfg, int32_t op, int32_t batch, int64_t rows, int64_t max_len_k)
{
    if (check_config(cfg) != QSA_OK || batch <= 0 || rows < 0) return 0;
    if (op == QSA_OP_DECODE)  // the even schedule runs below two rows per CTA
        return batch < 2 * kMaxEvenCtas ? even_workspace_bytes(batch, kMaxEvenCtas) : 0;
    if (op == QSA_OP_DECODE_PAGED) return even_workspace_bytes(batch, kMaxEvenCtas);
    if (op == QSA_OP_DECODE_MTP) return mtp_workspace_bytes(batch, cfg->budget_blocks);
    if (op == QSA_OP_INDEX_SELECT_PAGED)  // one score row per sequence
        return (size_t)batch * (max_len_k > 0 ? ((max_len_k - 1) / cfg->r + 3) / 4 * 4 + 4 : 4) * sizeof(float);
    if (op == QSA_OP_PREFILL) {
        const int nc = nchunks_of(cfg, max_len_k);
        return nc > 1 ? chunked_workspace_bytes(rows, nc) : 0;
    }
    if (op == QSA_OP_DENSE) return split_workspace_bytes(rows, dense_decode_nsplit(max_len_k, cfg->r));
    if (op == QSA_OP_INDEX_SELECT) {
        // prefill: samples, thresholds, candidate lists, fallback scratch; decode: one score row per row
        const size_t fused = index_select_workspace_bytes(rows, max_len_k, cfg->budget_blocks, cfg->r, num_sms());
        const int64_t ld = max_len_k > 0 ? ((max_len_k - 1) / cfg->r + 3) / 4 * 4 + 4 : 4;
        const size_t dec = decode_select_workspace_bytes(rows, ld, num_sms());
        return fused > dec ? fused : dec;
    }
    return 0;
}

qsa_status qsa_debug_inject(int32_t site)
{
#ifdef QSA_DEBUG_CHECKS
    if (site < 0 || site > 1) return QSA_ERR_INVALID_ARG;
    int v = site;
    return cudaMemcpyToSymbol(g_debug_fault_site, &v, sizeof(int)) == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
#else
    (void)site;
    return QSA_ERR_UNSUPPORTED;
#endif
}

qsa_status qsa_get_device_status(void *stream, int32_t *status, int32_t clear)
{
    if (status == nullptr) return QSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return QSA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return QSA_ERR_CUDA;
    *status = v;
    if (clear) {
        int z = 0;
        if (cudaMemcpyToSymbol(g_device_status, &z, sizeof(int)) != cudaSuccess) return QSA_ERR_CUDA;
    }
    return QSA_OK;
}

qsa_status qsa_compress_keys(const qsa_config *cfg, const qsa_bf16 *k_idx, const int32_t *cu_seqlens_k,
                             const int32_t *cu_blocks, int32_t batch, int64_t total_k, const int32_t *blk_begin,
                             int32_t max_new_blocks, qsa_bf16 *kc, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_compress_keys");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_k < 0 || cu_seqlens_k == nullptr || cu_blocks == nullptr) return QSA_ERR_INVALID_ARG;
    if (total_k == 0) return QSA_OK;
    if (k_idx == nullptr || kc == nullptr || !al16(k_idx) || !al16(kc)) return QSA_ERR_INVALID_ARG;
    if (blk_begin != nullptr && max_new_blocks <= 0) return QSA_ERR_INVALID_ARG;
    return cuda_status(launch_compress(bf(k_idx), cu_seqlens_k, cu_blocks, batch, total_k, blk_begin,
                                       max_new_blocks, cfg->r, (cfg->flags & QSA_COMPRESS_NO_NORM) == 0,
                                       cfg->rms_eps, bf(kc), static_cast<cudaStream_t>(stream), rope_of(cfg)));
}

qsa_status qsa_rope_queries(const qsa_config *cfg, qsa_bf16 *q_idx, const int32_t *cu_seqlens_q,
                            const int32_t *cu_seqlens_k, int32_t batch, int64_t total_q, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_rope_queries");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if ((cfg->flags & QSA_INDEX_ROPE) == 0) return QSA_ERR_INVALID_ARG;
    if (batch <= 0 || total_q < 0 || cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return QSA_ERR_INVALID_ARG;
    if (total_q == 0) return QSA_OK;
    if (q_idx == nullptr || !al16(q_idx)) return QSA_ERR_INVALID_ARG;
    __nv_bfloat16 *q = reinterpret_cast<__nv_bfloat16 *>(q_idx);
    return cuda_status(launch_rope_queries(q, q, cu_seqlens_q, cu_seqlens_k, batch, total_q, cfg->n_heads_idx,
                                           rope_of(cfg), static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_index_scores(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w, const qsa_bf16 *kc,
                            int64_t kc_rows, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            const int32_t *cu_blocks, int32_t batch, int64_t total_q, int32_t max_len_q,
                            int64_t row_begin, int64_t row_end, float *scores, int64_t ld, void *ws,
                            size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_index_scores");
    (void)ws;
    (void)ws_bytes;
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_q < 0 || kc_rows < 0 || ld <= 0 || max_len_q < 0) return QSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > total_q) return QSA_ERR_INVALID_ARG;
    if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr || cu_blocks == nullptr) return QSA_ERR_INVALID_ARG;
    if (row_end == row_begin || kc_rows == 0) return QSA_OK;
    if (q_idx == nullptr || w == nullptr || kc == nullptr || scores == nullptr || !al16(q_idx) || !al16(kc))
        return QSA_ERR_INVALID_ARG;
    IndexArgs a{bf(q_idx), w, bf(kc), kc_rows, cu_seqlens_q, cu_seqlens_k, cu_blocks, batch, total_q,
                row_begin, row_end, scores, ld, cfg->r};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (max_len_q == 1) return cuda_status(launch_index_rowwise(a, s));
    return cuda_status(launch_index_tc(a, s));
}

qsa_status qsa_index_select(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w, const qsa_bf16 *kc,
                            int64_t kc_rows, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                            const int32_t *cu_blocks, int32_t batch, int64_t total_q, int32_t max_len_q,
                            int64_t max_len_k, int64_t row_begin, int64_t row_end, int32_t *sel, void *ws,
                            size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_index_select");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_q < 0 || kc_rows < 0 || max_len_q < 0 || max_len_k < 0) return QSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > total_q) return QSA_ERR_INVALID_ARG;
    if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr || cu_blocks == nullptr) return QSA_ERR_INVALID_ARG;
    if (row_end == row_begin) return QSA_OK;
    if (q_idx == nullptr || w == nullptr || kc == nullptr || sel == nullptr || !al16(q_idx) || !al16(kc))
        return QSA_ERR_INVALID_ARG;
    const int64_t rows = row_end - row_begin;
    if (ws == nullptr || !al16(ws)) return QSA_ERR_WORKSPACE_TOO_SMALL;
    if (ws_bytes < qsa_workspace_size(cfg, QSA_OP_INDEX_SELECT, batch, rows, max_len_k))
        return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t ld = max_len_k > 0 ? ((max_len_k - 1) / cfg->r + 3) / 4 * 4 + 4 : 4;
    IndexArgs a{bf(q_idx), w, bf(kc), kc_rows, cu_seqlens_q, cu_seqlens_k, cu_blocks, batch, total_q,
                row_begin, row_end, static_cast<float *>(ws), ld, cfg->r};
    if (kc_rows == 0) {  // no complete block anywhere: every row keeps only its own block
        SelectArgs sa{static_cast<const float *>(ws), ld, cu_seqlens_q, cu_seqlens_k, batch, row_begin, row_end, sel,
                      cfg->budget_blocks, cfg->r};
        return cuda_status(launch_select(sa, s));
    }
    if (max_len_q == 1) {
        // decode rows: the hi-plane scan and the exact rescoring of each row's window
        // (the error bound needs RMSNorm'ed keys; without the norm, the exact scan)
        const bool refine = (cfg->flags & QSA_COMPRESS_NO_NORM) == 0;
        return cuda_status(launch_decode_index_select(a, cfg->budget_blocks, ws, num_sms(), refine, sel, s));
    }
    return cuda_status(launch_index_select(a, cfg->budget_blocks, ws, num_sms(), max_len_k, sel, s));
}

qsa_status qsa_compress_keys_paged(const qsa_config *cfg, const qsa_bf16 *k_idx_pages, qsa_bf16 *kc_pages,
                                   int64_t num_pages, int32_t page_size, const int32_t *block_table,
                                   int32_t max_pages, const int32_t *cu_seqlens_k, int32_t batch, int64_t max_len_k,
                                   const int32_t *blk_begin, int32_t max_new_blocks, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_compress_keys_paged");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || num_pages <= 0 || page_size <= 0 || max_pages <= 0 || max_len_k < 0 ||
        cu_seqlens_k == nullptr || block_table == nullptr)
        return QSA_ERR_INVALID_ARG;
    if (page_size % cfg->r != 0 || (blk_begin != nullptr && max_new_blocks <= 0)) return QSA_ERR_INVALID_ARG;
    if (num_pages * (int64_t)page_size >= ((int64_t)1 << 40)) return QSA_ERR_UNSUPPORTED;
    if (k_idx_pages == nullptr || kc_pages == nullptr || !al16(k_idx_pages) || !al16(kc_pages))
        return QSA_ERR_INVALID_ARG;
    PagedArgs p{num_pages, page_size, block_table, max_pages, cu_seqlens_k, batch, cfg->r};
    return cuda_status(launch_compress_paged(p, bf(k_idx_pages), bf(kc_pages), blk_begin, max_new_blocks, max_len_k,
                                             (cfg->flags & QSA_COMPRESS_NO_NORM) == 0, cfg->rms_eps,
                                             static_cast<cudaStream_t>(stream), rope_of(cfg)));
}

qsa_status qsa_index_select_paged(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w,
                                  const qsa_bf16 *kc_pages, int64_t num_pages, int32_t page_size,
                                  const int32_t *block_table, int32_t max_pages, const int32_t *cu_seqlens_k,
                                  int32_t batch, int64_t max_len_k, int32_t *sel, void *ws, size_t ws_bytes,
                                  void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_index_select_paged");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || batch > 65535 || num_pages <= 0 || page_size <= 0 || max_pages <= 0 || max_len_k <= 0 ||
        cu_seqlens_k == nullptr || block_table == nullptr)
        return QSA_ERR_INVALID_ARG;
    if (page_size % cfg->r != 0) return QSA_ERR_INVALID_ARG;
    if (q_idx == nullptr || w == nullptr || kc_pages == nullptr || sel == nullptr || !al16(q_idx) || !al16(kc_pages))
        return QSA_ERR_INVALID_ARG;
    const int64_t ld = ((max_len_k - 1) / cfg->r + 3) / 4 * 4 + 4;
    if (ws == nullptr || !al16(ws) || ws_bytes < (size_t)batch * ld * sizeof(float)) return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PagedArgs p{num_pages, page_size, block_table, max_pages, cu_seqlens_k, batch, cfg->r};
    float *scores = static_cast<float *>(ws);
    cudaError_t e = launch_index_paged(p, bf(q_idx), w, bf(kc_pages), scores, ld, s);
    if (e != cudaSuccess) return QSA_ERR_CUDA;
    SelectArgs sa{scores, ld, nullptr, cu_seqlens_k, batch, 0, batch, sel, cfg->budget_blocks, cfg->r};
    return cuda_status(launch_select(sa, s));
}

qsa_status qsa_select_blocks(const qsa_config *cfg, const float *scores, int64_t ld, const int32_t *cu_seqlens_q,
                             const int32_t *cu_seqlens_k, int32_t batch, int64_t row_begin, int64_t row_end,
                             int32_t *sel, void *ws, size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_select_blocks");
    (void)ws;
    (void)ws_bytes;
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || ld <= 0 || row_begin < 0 || row_end < row_begin) return QSA_ERR_INVALID_ARG;
    if (cu_seqlens_k == nullptr || cu_seqlens_q == nullptr) return QSA_ERR_INVALID_ARG;
    if (row_end == row_begin) return QSA_OK;
    if (scores == nullptr || sel == nullptr) return QSA_ERR_INVALID_ARG;
    SelectArgs a{scores, ld, cu_seqlens_q, cu_seqlens_k, batch, row_begin, row_end, sel, cfg->budget_blocks, cfg->r};
    return cuda_status(launch_select(a, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_sparse_attn_prefill(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k, const qsa_bf16 *v,
                                   const int32_t *sel, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                   int32_t batch, int64_t total_q, int64_t total_k, int64_t max_len_k,
                                   int64_t row_begin, int64_t row_end, qsa_bf16 *o, float *lse, void *ws,
                                   size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_sparse_attn_prefill");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_q < 0 || total_k < 0 || max_len_k < 0 || row_begin < 0 || row_end < row_begin ||
        row_end > total_q)
        return QSA_ERR_INVALID_ARG;
    if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return QSA_ERR_INVALID_ARG;
    if (row_end == row_begin) return QSA_OK;
    if (total_k == 0 || q == nullptr || k == nullptr || v == nullptr || sel == nullptr || o == nullptr ||
        !al16(q) || !al16(k) || !al16(v))
        return QSA_ERR_INVALID_ARG;
    AttnArgs a{bf(q), bf(k), bf(v), sel, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, row_begin, row_end,
               bf(o), lse, nullptr, 1, cfg->budget_blocks, cfg->r, cfg->softmax_scale};
    // the L2-blocked schedule when the keys span several chunks and the workspace allows it
    const int nc = nchunks_of(cfg, max_len_k);
    if (nc > 1 && ws != nullptr && al16(ws) && ws_bytes >= chunked_workspace_bytes(row_end - row_begin, nc)) {
        a.ws = static_cast<float *>(ws);
        a.nchunks = nc;
        a.chunk_blocks = cfg->kv_chunk_blocks;
    }
    return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_sparse_attn_decode(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_cache,
                                  const qsa_bf16 *v_cache, const int32_t *cu_seqlens_k, int32_t batch,
                                  int64_t total_k, const int32_t *sel, qsa_bf16 *o, float *lse, void *ws,
                                  size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_sparse_attn_decode");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_k <= 0 || cu_seqlens_k == nullptr) return QSA_ERR_INVALID_ARG;
    if (q == nullptr || k_cache == nullptr || v_cache == nullptr || sel == nullptr || o == nullptr ||
        !al16(q) || !al16(k_cache) || !al16(v_cache))
        return QSA_ERR_INVALID_ARG;
    // below two rows per CTA the batch's tiles are spread evenly over the CTAs (rows cut
    // in pieces, merged by a second kernel); above, one CTA per row at a time balances
    const int grid = even_grid();
    const bool even = batch < 2 * grid;
    if (even) {
        if (ws == nullptr) return QSA_ERR_WORKSPACE_TOO_SMALL;
        if (ws_bytes < even_workspace_bytes(batch, grid)) return QSA_ERR_WORKSPACE_TOO_SMALL;
        if (!al16(ws)) return QSA_ERR_INVALID_ARG;
    }
    AttnArgs a{bf(q), bf(k_cache), bf(v_cache), sel, nullptr, cu_seqlens_k, batch, batch, total_k, 0, batch,
               bf(o), lse, even ? static_cast<float *>(ws) : nullptr, 1, cfg->budget_blocks, cfg->r,
               cfg->softmax_scale};
    a.even = even ? 1 : 0;
    return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_sparse_attn_decode_window(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_local,
                                         const qsa_bf16 *v_local, const int32_t *cu_seqlens_k, int32_t batch,
                                         int64_t total_k_local, const int64_t *tok_local, const int32_t *blk_lo,
                                         const int32_t *blk_hi, const int32_t *sel, qsa_bf16 *o, float *lse,
                                         void *ws, size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_sparse_attn_decode_window");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_k_local <= 0 || cu_seqlens_k == nullptr || tok_local == nullptr || blk_lo == nullptr ||
        blk_hi == nullptr)
        return QSA_ERR_INVALID_ARG;
    if (q == nullptr || k_local == nullptr || v_local == nullptr || sel == nullptr || o == nullptr || lse == nullptr ||
        !al16(q) || !al16(k_local) || !al16(v_local))
        return QSA_ERR_INVALID_ARG;
    const int grid = even_grid();
    if (batch >= 2 * grid) return QSA_ERR_UNSUPPORTED;  // the even schedule only
    if (ws == nullptr) return QSA_ERR_WORKSPACE_TOO_SMALL;
    if (ws_bytes < even_workspace_bytes(batch, grid)) return QSA_ERR_WORKSPACE_TOO_SMALL;
    if (!al16(ws)) return QSA_ERR_INVALID_ARG;
    AttnArgs a{bf(q), bf(k_local), bf(v_local), sel, nullptr, cu_seqlens_k, batch, batch, total_k_local, 0, batch,
               bf(o), lse, static_cast<float *>(ws), 1, cfg->budget_blocks, cfg->r, cfg->softmax_scale};
    a.even = 1;
    a.tok_local = tok_local;
    a.blk_lo = blk_lo;
    a.blk_hi = blk_hi;
    return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_merge_attn_states(const qsa_config *cfg, const qsa_bf16 *o_parts, const float *lse_parts,
                                 int32_t parts, int64_t rows, qsa_bf16 *o, float *lse, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_merge_attn_states");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (parts <= 0 || rows < 0) return QSA_ERR_INVALID_ARG;
    if (rows == 0) return QSA_OK;
    if (o_parts == nullptr || lse_parts == nullptr || o == nullptr) return QSA_ERR_INVALID_ARG;
    return cuda_status(launch_merge_states(bf(o_parts), lse_parts, parts, rows,
                                           reinterpret_cast<__nv_bfloat16 *>(o), lse,
                                           static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_sparse_attn_decode_paged(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_pages,
                                        const qsa_bf16 *v_pages, int64_t num_pages, int32_t page_size,
                                        const int32_t *block_table, int32_t max_pages,
                                        const int32_t *cu_seqlens_k, int32_t batch, const int32_t *sel,
                                        qsa_bf16 *o, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_sparse_attn_decode_paged");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || num_pages <= 0 || page_size <= 0 || max_pages <= 0 || cu_seqlens_k == nullptr ||
        block_table == nullptr)
        return QSA_ERR_INVALID_ARG;
    if (page_size % cfg->r != 0) return QSA_ERR_INVALID_ARG;
    if (num_pages * (int64_t)page_size * cfg->n_heads_kv >= ((int64_t)1 << 31)) return QSA_ERR_UNSUPPORTED;
    if (q == nullptr || k_pages == nullptr || v_pages == nullptr || sel == nullptr || o == nullptr || !al16(q) ||
        !al16(k_pages) || !al16(v_pages))
        return QSA_ERR_INVALID_ARG;
    const int grid = even_grid();
    if (ws == nullptr || ws_bytes < even_workspace_bytes(batch, grid)) return QSA_ERR_WORKSPACE_TOO_SMALL;
    if (!al16(ws)) return QSA_ERR_INVALID_ARG;
    AttnArgs a{bf(q), bf(k_pages), bf(v_pages), sel, nullptr, cu_seqlens_k, batch, batch, num_pages * page_size, 0,
               batch, bf(o), lse, static_cast<float *>(ws), 1, cfg->budget_blocks, cfg->r, cfg->softmax_scale};
    a.even = 1;
    a.block_table = block_table;
    a.page_size = page_size;
    a.max_pages = max_pages;
    return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_index_select_mtp(const qsa_config *cfg, const qsa_bf16 *q_idx, const float *w, const qsa_bf16 *kc,
                                int64_t kc_rows, const int32_t *cu_seqlens_k, const int32_t *cu_blocks,
                                int32_t batch, int32_t next_n, int64_t max_len_k, int32_t *sel, void *ws,
                                size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_index_select_mtp");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || kc_rows < 0 || max_len_k <= 0 || next_n < 1 || next_n > 4 || cu_seqlens_k == nullptr ||
        cu_blocks == nullptr)
        return QSA_ERR_INVALID_ARG;
    if (cfg->budget_blocks < 2) return QSA_ERR_UNSUPPORTED;  // two own blocks may be forced
    if (q_idx == nullptr || w == nullptr || sel == nullptr || (kc_rows > 0 && kc == nullptr) || !al16(q_idx) ||
        (kc != nullptr && !al16(kc)))
        return QSA_ERR_INVALID_ARG;
    if (ws == nullptr || !al16(ws) ||
        ws_bytes < qsa_workspace_size(cfg, QSA_OP_INDEX_SELECT, batch, batch, max_len_k))
        return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t ld = ((max_len_k - 1) / cfg->r + 3) / 4 * 4 + 4;
    // the one query row of each sequence whose scores serve the step: its last (t = L - 1)
    const int32_t *cu_q = nullptr;
    IndexArgs a{bf(q_idx), w, bf(kc), kc_rows, cu_q, cu_seqlens_k, cu_blocks, batch, batch, 0, batch,
                static_cast<float *>(ws), ld, cfg->r};
    if (kc_rows == 0) {
        SelectArgs sa{static_cast<const float *>(ws), ld, nullptr, cu_seqlens_k, batch, 0, batch, sel,
                      cfg->budget_blocks, cfg->r};
        sa.next_n = next_n;
        return cuda_status(launch_select(sa, s));
    }
    const bool refine = (cfg->flags & QSA_COMPRESS_NO_NORM) == 0;
    return cuda_status(launch_decode_index_select(a, cfg->budget_blocks, ws, num_sms(), refine, sel, s, next_n));
}

qsa_status qsa_sparse_attn_decode_mtp(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_cache,
                                      const qsa_bf16 *v_cache, const int32_t *cu_seqlens_k, int32_t batch,
                                      int64_t total_k, int32_t next_n, const int32_t *sel, qsa_bf16 *o, float *lse,
                                      void *ws, size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_sparse_attn_decode_mtp");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_k <= 0 || next_n < 1 || next_n > 4 || cu_seqlens_k == nullptr) return QSA_ERR_INVALID_ARG;
    if (q == nullptr || k_cache == nullptr || v_cache == nullptr || sel == nullptr || o == nullptr || !al16(q) ||
        !al16(k_cache) || !al16(v_cache) || !al16(o))
        return QSA_ERR_INVALID_ARG;
    const size_t need = mtp_workspace_bytes(batch, cfg->budget_blocks);
    if (need > 0 && (ws == nullptr || ws_bytes < need)) return QSA_ERR_WORKSPACE_TOO_SMALL;
    if (need > 0 && !al16(ws)) return QSA_ERR_INVALID_ARG;
    AttnArgs a{bf(q), bf(k_cache), bf(v_cache), sel, nullptr, cu_seqlens_k, batch, batch, total_k, 0, batch,
               bf(o), lse, static_cast<float *>(ws), 1, cfg->budget_blocks, cfg->r, cfg->softmax_scale};
    return cuda_status(launch_sparse_mtp(a, next_n, static_cast<cudaStream_t>(stream)));
}

qsa_status qsa_dense_attn_prefill(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k, const qsa_bf16 *v,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int32_t batch,
                                  int64_t total_q, int64_t total_k, int32_t max_len_q, int64_t max_len_k,
                                  qsa_bf16 *o, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_dense_attn_prefill");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_q < 0 || total_k < 0 || max_len_q < 0 || max_len_k < 0 || cu_seqlens_q == nullptr ||
        cu_seqlens_k == nullptr)
        return QSA_ERR_INVALID_ARG;
    if (total_q == 0) return QSA_OK;
    if (total_k == 0 || q == nullptr || k == nullptr || v == nullptr || o == nullptr || !al16(q) || !al16(k) ||
        !al16(v))
        return QSA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (max_len_q == 1) {
        // one query per sequence: split-K flash decoding over every block (HBM-bound)
        const int nsplit = dense_decode_nsplit(max_len_k, cfg->r);
        if (nsplit > 1 && (ws == nullptr || ws_bytes < split_workspace_bytes(total_q, nsplit)))
            return QSA_ERR_WORKSPACE_TOO_SMALL;
        if (nsplit > 1 && !al16(ws)) return QSA_ERR_INVALID_ARG;
        const int kb = (int)((max_len_k + cfg->r - 1) / cfg->r);
        AttnArgs a{bf(q), bf(k), bf(v), nullptr, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, 0, total_q,
                   bf(o), lse, static_cast<float *>(ws), nsplit, kb > 0 ? kb : 1, cfg->r, cfg->softmax_scale};
        return cuda_status(launch_sparse_attn(a, s));
    }
    DenseArgs a{bf(q), bf(k), bf(v), cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_len_q, bf(o), lse,
                cfg->softmax_scale};
    return cuda_status(launch_dense_attn(a, s));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode with library-held scratch.  For callers that cannot allocate device
// memory while decoding (a pool that has reserved all free memory up front, a
// plain C host without a device allocator): the partial softmax states live in
// a fixed array of the library's device image instead of a caller workspace.
// Every GPU that loads the library holds the array until the process exits;
// every call on a device shares it, so calls whose kernels overlap on the GPU
// race.  Nothing in it needs to start at zero: each call writes every partial
// state (a neutral one for an empty split) before the merge kernel reads it.

static __device__ __align__(256) float g_decode_scratch[QSA_STATIC_SCRATCH_BYTES / sizeof(float)];

namespace {

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxScratchDevices];  // device address of g_decode_scratch, per device ordinal

// Set-up, once per device, with that device current: the array's device
// address.  The first call on a device therefore does this lookup, which
// belongs before any stream capture.
qsa_status decode_scratch(float **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return QSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxScratchDevices) return QSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return QSA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = static_cast<float *>(g_scratch_ptr[dev]);
    return QSA_OK;
}

}  // namespace

extern "C" {

qsa_status qsa_sparse_attn_decode_static_scratch(const qsa_config *cfg, const qsa_bf16 *q, const qsa_bf16 *k_cache,
                                                 const qsa_bf16 *v_cache, const int32_t *cu_seqlens_k, int32_t batch,
                                                 int64_t total_k, const int32_t *sel, qsa_bf16 *o, float *lse,
                                                 void *stream)
{
    const qsa::NvtxRange nvtx_range("qsa_sparse_attn_decode_static_scratch");
    qsa_status st = check_config(cfg);
    if (st != QSA_OK) return st;
    if (batch <= 0 || total_k <= 0 || cu_seqlens_k == nullptr) return QSA_ERR_INVALID_ARG;
    if (q == nullptr || k_cache == nullptr || v_cache == nullptr || sel == nullptr || o == nullptr ||
        !al16(q) || !al16(k_cache) || !al16(v_cache))
        return QSA_ERR_INVALID_ARG;
    float *scratch = nullptr;
    st = decode_scratch(&scratch);
    if (st != QSA_OK) return st;
    const int grid = even_grid();
    const bool even = batch < 2 * grid;
    if (even && even_workspace_bytes(batch, grid) > (size_t)QSA_STATIC_SCRATCH_BYTES) return QSA_ERR_SCRATCH_LIMIT;
    AttnArgs a{bf(q), bf(k_cache), bf(v_cache), sel, nullptr, cu_seqlens_k, batch, batch, total_k, 0, batch,
               bf(o), lse, even ? scratch : nullptr, 1, cfg->budget_blocks, cfg->r, cfg->softmax_scale};
    a.even = even ? 1 : 0;
    return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
