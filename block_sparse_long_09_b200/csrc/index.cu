// index.cu -- QSA lightweight MQA indexer.
//
// Indexer equation of "On the Design of Qwen3.8 Next Architecture" (reading
// notes, section 6), with one weight per (query, indexer head):
//   S[t, b] = sum_{h<4} w[t, h] * ReLU(<q_idx[t, h, :], kc[b, :]>),  b < b_t = floor(t / r)
// 4 query heads share one key head of dim 128 ("Model Summary" table), so the
// cost is O(n^2 / r) (the section's complexity equation).
//
// Prefill path (index_tc_kernel): a causal GEMM on the 5th-generation tensor
// cores.  A CTA owns 64 consecutive query rows = 2 x 128 A-rows (token-major,
// head-minor, exactly the q_idx memory order), loaded once by TMA.  It walks
// the kc blocks below its causal bound in N-tiles of 128 blocks; kc holds a
// compensated bf16 pair (hi, lo) per value, and both planes are multiplied
// into the same fp32 accumulator:
//   warp 0      TMA producer (kc hi+lo tiles, 2-stage ring, 128-byte swizzle)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer: two M128 N128
//               accumulators (one per 32-row sub-tile) share each kc tile, so the
//               L2 traffic of kc is halved against 32-row tiles
//   warps 2..9  epilogue: tcgen05.ld of the fp32 accumulators (double-buffered in
//               TMEM -- all 512 columns -- so the next tile's MMAs overlap), ReLU
//               * w, a 4-lane butterfly that sums the heads while scattering
//               columns, 128-byte-swizzled staging in shared memory and 32 x 32
//               TMA bulk stores of the scores (scattered per-thread stores would
//               saturate the L1 store path).  Tiles that straddle two sequences
//               fall back to masked per-thread stores.
// Tiles above the diagonal are never issued; heavy (late) row tiles launch first.
//
// Decode path (index_rowwise_kernel): one query row per sequence is a GEMV over
// the kc cache -- HBM-bound, so it runs on CUDA cores: each warp streams 8 kc
// rows with coalesced 8-byte loads, keeps its 4 heads' query slice in
// registers, adds the hi and lo planes of kc in fp32, and reduces the 32
// (block, head) partial dots with a 5-step butterfly reduce-scatter.
#include "kernels.cuh"

namespace qsa {

namespace {

// ------------------------------------------------------------------ tcgen05 path
constexpr int kTokTile = 64;                  // query rows per CTA
constexpr int kSubTok = 32;                   // query rows per A sub-tile
constexpr int kBM = kSubTok * 4;              // A rows of a sub-tile (token x head) = MMA M
constexpr int kBN = 128;                      // kc blocks per N tile
constexpr int kIdxDim = 128;
constexpr int kStages = 2;
constexpr int kChunkA = kBM * 128;            // 16 KB: one 64-column swizzled chunk of a sub-tile
constexpr int kChunkB = kBN * 128;            // 16 KB
constexpr int kABytes = 2 * 2 * kChunkA;      // 64 KB: two sub-tiles
constexpr int kBBytes = 4 * kChunkB;          // 64 KB per stage: hi and lo planes
constexpr int kStgChunk = kSubTok * 128;      // 4 KB: 32 rows x 32 fp32 scores, swizzled
constexpr int kStgBytes = 2 * 4 * kStgChunk;  // 32 KB: 2 sub-tiles x 4 column groups
constexpr int kIdxThreads = 320;              // producer, MMA, 8 epilogue warps
constexpr uint32_t kAccCols = 512;            // 2 buffers x 2 sub-tiles x 128 columns

struct IdxShared {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t a_full;
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};

constexpr int kIdxSmem = kABytes + kStages * kBBytes + kStgBytes + (int)sizeof(IdxShared) + 1024;

struct Segment {
    int s;
    int64_t seg_begin, seg_end;  // packed rows of this tile that belong to sequence s
    int64_t pos_offset;          // t = pos_offset + (i - cu_q[s])
    int64_t kc_base;
    int n_tiles;
};

// Iterates the (sequence, N-tile) work of a row tile identically in every role.
struct SegIter {
    const int32_t *cu_q, *cu_k, *cu_blocks;
    int batch, r;
    int64_t m0, m1;
    int s;
    __device__ bool next(Segment &seg)
    {
        while (s < batch && (int64_t)cu_q[s] < m1) {
            const int cs = s++;
            const int64_t q0 = cu_q[cs], q1 = cu_q[cs + 1];
            const int64_t b = q0 > m0 ? q0 : m0;
            const int64_t e = q1 < m1 ? q1 : m1;
            if (e <= b) continue;
            const int64_t Lq = q1 - q0, Lk = (int64_t)cu_k[cs + 1] - cu_k[cs];
            seg.s = cs;
            seg.seg_begin = b;
            seg.seg_end = e;
            seg.pos_offset = Lk - Lq;
            seg.kc_base = cu_blocks[cs];
            const int64_t t_last = (Lk - Lq) + (e - 1 - q0);
            const int64_t bt_max = t_last >= 0 ? t_last / r : 0;
            seg.n_tiles = (int)((bt_max + kBN - 1) / kBN);
            if (seg.n_tiles == 0) continue;
            return true;
        }
        return false;
    }
};

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t x, int32_t y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void sub_bar(int sub) { asm volatile("bar.sync %0, 128;" ::"r"(2 + sub) : "memory"); }

__global__ void __launch_bounds__(kIdxThreads, 1)
index_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
                const __grid_constant__ CUtensorMap map_s, int use_tma_store,
                const float *__restrict__ w, const int32_t *__restrict__ cu_q,
                const int32_t *__restrict__ cu_k, const int32_t *__restrict__ cu_blocks, int batch,
                int64_t row_begin, int64_t row_end, float *__restrict__ scores, int64_t ld, int r)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kABytes;
    uint8_t *sStg = sB + kStages * kBBytes;
    IdxShared *sh = reinterpret_cast<IdxShared *>(sStg + kStgBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntile_rows = (row_end - row_begin + kTokTile - 1) / kTokTile;
    const int64_t tile = ntile_rows - 1 - blockIdx.x;  // heavy (late) tiles first
    const int64_t m0 = row_begin + tile * kTokTile;
    const int64_t m1 = (m0 + kTokTile < row_end) ? m0 + kTokTile : row_end;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sh->full[i], 1);
            mbar_init(&sh->empty[i], 1);
        }
        mbar_init(&sh->a_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->acc_full[i], 1);
            mbar_init(&sh->acc_empty[i], 8);
        }
        sh->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, kAccCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    volatile int *abort_flag = &sh->abort_flag;

    const int s0 = find_seq(cu_q, batch, m0);
    // one sequence covers the whole tile: whole 32 x 32 score boxes can be stored by TMA
    const bool single = use_tma_store && (int64_t)cu_q[s0 + 1] >= m1;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (elect_one()) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_kc);
            mbar_arrive_expect_tx(&sh->a_full, kABytes);
            for (int sub = 0; sub < 2; ++sub)
                for (int c = 0; c < 2; ++c)
                    tma_load_2d(sA + (sub * 2 + c) * kChunkA, &map_q, &sh->a_full, c * 64,
                                (int32_t)((m0 + sub * kSubTok) * 4));
            SegIter it{cu_q, cu_k, cu_blocks, batch, r, m0, m1, s0};
            Segment seg;
            uint32_t k = 0;
            bool ok = true;
            while (ok && it.next(seg)) {
                for (int n = 0; n < seg.n_tiles; ++n, ++k) {
                    const uint32_t st = k % kStages, round = k / kStages;
                    if (!mbar_wait(&sh->empty[st], (round & 1) ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&sh->full[st], kBBytes);
                    const int32_t y = (int32_t)(seg.kc_base + (int64_t)n * kBN);
                    for (int c = 0; c < 4; ++c)
                        tma_load_2d(sB + st * kBBytes + c * kChunkB, &map_kc, &sh->full[st], c * 64, y);
                }
            }
            if (!ok) {
                for (uint32_t j = (k > kStages ? k - kStages : 0); j < k; ++j)
                    mbar_wait(&sh->full[j % kStages], (j / kStages) & 1, nullptr);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
            const uint32_t a_addr = smem_u32(sA), b_addr = smem_u32(sB);
            bool ok = mbar_wait(&sh->a_full, 0, abort_flag);
            SegIter it{cu_q, cu_k, cu_blocks, batch, r, m0, m1, s0};
            Segment seg;
            uint32_t k = 0;
            while (ok && it.next(seg)) {
                for (int n = 0; n < seg.n_tiles; ++n, ++k) {
                    const uint32_t st = k % kStages, round = k / kStages;
                    const uint32_t acc = k & 1, use = k >> 1;
                    if (!mbar_wait(&sh->acc_empty[acc], (use & 1) ^ 1, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&sh->full[st], round & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {
                        const uint32_t d = tmem + (acc * 2 + sub) * kBN;
#pragma unroll
                        for (int ks = 0; ks < 2 * kIdxDim / 16; ++ks) {  // hi plane, then lo plane
                            const int ka = ks & 7;                    // k-step within the 128 dims
                            const uint32_t koff = (ka & 3) * 32;
                            const uint64_t ad = sdesc_sw128(a_addr + (sub * 2 + (ka >> 2)) * kChunkA + koff, 16, 1024);
                            const uint64_t bd = sdesc_sw128(b_addr + st * kBBytes + (ks >> 2) * kChunkB + koff, 16, 1024);
                            mma_bf16_ss(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(&sh->empty[st]);
                    mma_commit(&sh->acc_full[acc]);
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 2..9) ----------------
        const int ew = warp - 2;
        const int sub = ew >> 2;                   // A sub-tile
        const int quad = warp & 3;                 // TMEM lane quadrant this warp may read
        const int row_in_sub = quad * 8 + (lane >> 2);
        const int head = lane & 3;
        const int64_t i = m0 + sub * kSubTok + row_in_sub;  // packed query row of this lane
        const float wv = (i < m1) ? __ldg(w + i * 4 + head) : 0.f;
        const bool b0 = lane & 1, b1 = (lane >> 1) & 1;
        const int col_sub = (b0 ? 16 : 0) + (b1 ? 8 : 0);
        const bool vec_ok = (ld & 3) == 0;
        const bool store_thread = (ew & 3) == 0 && lane == 0;  // issues this sub-tile's TMA stores
        uint8_t *stg = sStg + sub * 4 * kStgChunk;
        const uint32_t stg_row = (uint32_t)row_in_sub * 128;
        const int unit0 = col_sub >> 2;            // first 16-byte unit of the 8 values

        SegIter it{cu_q, cu_k, cu_blocks, batch, r, m0, m1, s0};
        Segment seg;
        uint32_t k = 0;
        bool ok = true;
        while (ok && it.next(seg)) {
            const bool row_in_seg = (i >= seg.seg_begin && i < seg.seg_end);
            const int64_t t = seg.pos_offset + (i - cu_q[seg.s]);
            int64_t bt = row_in_seg ? t / r : 0;
            if (bt > ld) {
                if (lane == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
                bt = ld;
            }
            float *srow = scores + (i - row_begin) * ld;
            for (int n = 0; n < seg.n_tiles; ++n, ++k) {
                const uint32_t acc = k & 1, use = k >> 1;
                if (!mbar_wait(&sh->acc_full[acc], use & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (single) {
                    if (store_thread) bulk_wait_read0();  // staging free again
                    sub_bar(sub);
                }
#pragma unroll 1
                for (int c = 0; c < kBN / 32; ++c) {
                    float v[32];
                    tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + (acc * 2 + sub) * kBN + c * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = wv * fmaxf(v[j], 0.f);
                    // butterfly over the 4 head lanes: sum heads, scatter columns
                    float h16[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float send = b0 ? v[j] : v[j + 16];
                        const float keep = b0 ? v[j + 16] : v[j];
                        h16[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                    }
                    float h8[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float send = b1 ? h16[j] : h16[j + 8];
                        const float keep = b1 ? h16[j + 8] : h16[j];
                        h8[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    }
                    if (single) {
                        // 128-byte swizzled staging row: 16-byte unit u lands at u ^ (row & 7)
                        uint8_t *base = stg + c * kStgChunk + stg_row;
                        const int sw = row_in_sub & 7;
                        *reinterpret_cast<float4 *>(base + (((unit0) ^ sw) << 4)) = make_float4(h8[0], h8[1], h8[2], h8[3]);
                        *reinterpret_cast<float4 *>(base + (((unit0 + 1) ^ sw) << 4)) = make_float4(h8[4], h8[5], h8[6], h8[7]);
                    } else if (row_in_seg) {
                        const int64_t bcol = (int64_t)n * kBN + c * 32 + col_sub;
                        if (vec_ok && bcol + 8 <= bt) {
                            float4 *dst = reinterpret_cast<float4 *>(srow + bcol);
                            dst[0] = make_float4(h8[0], h8[1], h8[2], h8[3]);
                            dst[1] = make_float4(h8[4], h8[5], h8[6], h8[7]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (bcol + j < bt) srow[bcol + j] = h8[j];
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh->acc_empty[acc]);
                if (single) {
                    fence_proxy_async_smem();
                    sub_bar(sub);
                    if (store_thread) {
                        const int32_t y = (int32_t)(m0 + sub * kSubTok - row_begin);
                        for (int c = 0; c < 4; ++c)
                            tma_store_2d(&map_s, stg + c * kStgChunk, n * kBN + c * 32, y);
                        bulk_commit();
                    }
                }
            }
        }
        if (store_thread) bulk_wait0();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kAccCols);
    }
}

// ------------------------------------------------------------------ row-wise path
constexpr int kRowWarps = 8;
constexpr int kRowChunk = 1024;  // kc blocks per CTA

__global__ void __launch_bounds__(kRowWarps * 32)
index_rowwise_kernel(const __nv_bfloat16 *__restrict__ q_idx, const float *__restrict__ w,
                     const __nv_bfloat16 *__restrict__ kc, const int32_t *__restrict__ cu_q,
                     const int32_t *__restrict__ cu_k, const int32_t *__restrict__ cu_blocks,
                     int batch, int64_t row_begin, float *__restrict__ scores, int64_t ld, int r)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t i = row_begin + blockIdx.y;
    const int s = find_seq(cu_q, batch, i);
    const int64_t Lq = (int64_t)cu_q[s + 1] - cu_q[s];
    const int64_t Lk = (int64_t)cu_k[s + 1] - cu_k[s];
    const int64_t t = (Lk - Lq) + (i - cu_q[s]);
    int64_t bt = t >= 0 ? t / r : 0;
    if (bt > ld || (int64_t)cu_blocks[s + 1] - cu_blocks[s] != Lk / r) {
        if (threadIdx.x == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        if ((int64_t)cu_blocks[s + 1] - cu_blocks[s] != Lk / r) return;
        bt = ld;
    }
    const int64_t c0 = (int64_t)blockIdx.x * kRowChunk;
    const int64_t c1 = (c0 + kRowChunk < bt) ? c0 + kRowChunk : bt;
    if (c0 >= c1) return;

    // this lane's slice of the 4 query heads: dims 4 lane .. 4 lane + 3
    float q[4][4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        uint2 raw = *reinterpret_cast<const uint2 *>(q_idx + (i * 4 + h) * 128 + lane * 4);
        float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.x));
        float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.y));
        q[h][0] = a.x; q[h][1] = a.y; q[h][2] = b.x; q[h][3] = b.y;
    }
    const float wv = __ldg(w + i * 4 + (lane & 3));
    const __nv_bfloat16 *kbase = kc + (int64_t)cu_blocks[s] * 256 + lane * 4;
    float *srow = scores + (int64_t)blockIdx.y * ld;

    for (int64_t b0 = c0 + warp * 8; b0 < c1; b0 += kRowWarps * 8) {
        uint2 raw[8], rlo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t b = b0 + j;
            const bool in = b < c1;
            raw[j] = in ? __ldg(reinterpret_cast<const uint2 *>(kbase + b * 256)) : make_uint2(0u, 0u);
            rlo[j] = in ? __ldg(reinterpret_cast<const uint2 *>(kbase + b * 256 + 128)) : make_uint2(0u, 0u);
        }
        float v[32];  // v[j * 4 + h] = partial dot of block b0 + j with head h
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw[j].x));
            float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw[j].y));
            const float2 al = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&rlo[j].x));
            const float2 bl = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&rlo[j].y));
            a.x += al.x; a.y += al.y; b.x += bl.x; b.y += bl.y;
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
    }
}

}  // namespace

cudaError_t launch_index_tc(const IndexArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0 || a.kc_rows <= 0) return cudaSuccess;
    CUtensorMap mq, mk, ms;
    if (!make_tmap_2d(&mq, a.q_idx, 128, (uint64_t)a.total_q * 4, 256, 64, kBM)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&mk, a.kc, 256, (uint64_t)a.kc_rows, 512, 64, kBN)) return cudaErrorInvalidValue;
    // the scores of this call as an fp32 [rows, ld] tensor for 32 x 32 TMA stores (needs ld % 4 == 0)
    int use_tma = ((a.ld & 3) == 0) && make_tmap_2d_f32(&ms, a.scores, (uint64_t)a.ld, (uint64_t)rows,
                                                       (uint64_t)a.ld * 4, 32, 32);
    if (!use_tma) ms = mq;  // unused
    {
        const cudaError_t e = set_smem_attr_once(reinterpret_cast<const void *>(index_tc_kernel), kIdxSmem);
        if (e != cudaSuccess) return e;
    }
    const int64_t tiles = (rows + kTokTile - 1) / kTokTile;
    index_tc_kernel<<<(unsigned)tiles, kIdxThreads, kIdxSmem, stream>>>(
        mq, mk, ms, use_tma, a.w, a.cu_q, a.cu_k, a.cu_blocks, a.batch, a.row_begin, a.row_end, a.scores, a.ld,
        a.r);
    return cudaGetLastError();
}

cudaError_t launch_index_rowwise(const IndexArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0 || a.kc_rows <= 0) return cudaSuccess;
    const int64_t chunks = (a.ld + kRowChunk - 1) / kRowChunk;
    for (int64_t done = 0; done < rows; done += 65535) {
        const int64_t n = rows - done < 65535 ? rows - done : 65535;
        dim3 grid((unsigned)chunks, (unsigned)n);
        index_rowwise_kernel<<<grid, kRowWarps * 32, 0, stream>>>(
            a.q_idx, a.w, a.kc, a.cu_q, a.cu_k, a.cu_blocks, a.batch, a.row_begin + done,
            a.scores + done * a.ld, a.ld, a.r);
    }
    return cudaGetLastError();
}

}  // namespace qsa
