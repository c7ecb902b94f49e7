// index.cu -- QSA lightweight MQA indexer.
//
// Indexer equation of "On the Design of Qwen3.8 Next Architecture" (reading
// notes, section 6), with one weight per (query, indexer head):
//   S[t, b] = sum_{h<4} w[t, h] * ReLU(<q_idx[t, h, :], kc[b, :]>),  b < b_t = floor(t / r)
// 4 query heads share one key head of dim 128 ("Model Summary" table), so the
// cost is O(n^2 / r) (the section's complexity equation).
//
// Prefill path (index_tc_kernel): a causal GEMM on the 5th-generation tensor
// cores, "swap AB": the compressed keys are the MMA's M side and the CTA's 64
// query rows x 4 heads (256 rows, the q_idx memory order) its N side, so one
// M128 N256 accumulator holds, in TMEM lane b, all 4 heads of all 64 rows
// against kc block b.  The head sum is then local to a thread and the scores
// of a row leave as coalesced 128-byte runs of consecutive blocks.
//   warp 0       TMA producer: the q tile once (64 rows x 4 heads x 128), then
//                kc tiles of 128 blocks (hi and lo planes) through a 2-stage ring
//                (128-byte swizzle)
//   warp 1       TMEM allocator + single-thread tcgen05.mma issue (kind::f16, bf16
//                operands, fp32 accumulation): kc is a compensated bf16 pair, so
//                every k-step multiplies q by the hi plane and then by the lo plane
//                into the same accumulator; two 256-column accumulators in TMEM so
//                the next tile's MMAs overlap the epilogue
//   warps 2..17  the epilogue: tcgen05.ld of the thread's 16 rows x 4 heads,
//                ReLU * w, the head sum, and what the mode asks for (below)
// Tiles above the diagonal are never issued; heavy (late) row tiles launch first.
//
// Decode path (index_rowwise_kernel): one query row per sequence is a GEMV over
// the kc cache -- HBM-bound, so it runs on CUDA cores: each warp streams 8 kc
// rows with coalesced 8-byte loads, keeps its 4 heads' query slice in
// registers, and reduces the 32 (block, head) partial dots with a 5-step
// butterfly reduce-scatter.
#include <type_traits>

#include "kernels.cuh"

namespace qsa {

namespace {

// ------------------------------------------------------------------ tcgen05 path
constexpr int kTokTile = 64;                  // query rows per CTA
constexpr int kQRowsT = kTokTile * 4;         // N: rows x heads = 256
constexpr int kBM = 128;                      // M: kc blocks per tile
constexpr int kIdxDim = 128;
constexpr int kStages = 2;
constexpr int kChunkQ = kQRowsT * 128;        // 32 KB: one 64-dim swizzled chunk of the q tile
constexpr int kQBytes = 2 * kChunkQ;          // 64 KB
constexpr int kChunkKc = kBM * 128;           // 16 KB: one 64-dim chunk of one plane
constexpr int kKcBytes = 4 * kChunkKc;        // 64 KB per stage: hi and lo planes
constexpr int kEpiWarps = 16;                 // 4 per TMEM lane quadrant
constexpr int kIdxThreads = 64 + kEpiWarps * 32;
constexpr uint32_t kAccCols = 512;            // 2 buffers x 256 columns

struct IdxShared {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t q_full;      // the q tile landed
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
    // w of the tile's rows, by row pairs (2p, 2p + 1): {w[2p][0], w[2p+1][0], w[2p][1], w[2p+1][1]},
    // then the same for heads 2, 3 -- each float2 an operand of the packed fp32x2 epilogue
    alignas(16) float wq[kQRowsT];
    alignas(16) float theta[kTokTile];  // emit mode: the rows' thresholds; read as float4
    int seg_len[kEpiWarps][16];  // emit mode: each epilogue warp's list-segment lengths
};

static_assert(offsetof(IdxShared, wq) % 16 == 0, "the weight table is read as float4");
static_assert(offsetof(IdxShared, theta) % 16 == 0, "the thresholds are read as float4");
constexpr int kIdxSmem = kQBytes + kStages * kKcBytes + (int)sizeof(IdxShared) + 1024;
static_assert(kIdxSmem <= 232448, "shared memory of one CTA");

struct Segment {
    int s;
    int64_t seg_begin, seg_end;  // packed rows of this tile that belong to sequence s
    int64_t pos_offset;          // t = pos_offset + (i - cu_q[s])
    int64_t q0;                  // cu_q[s]
    int64_t kc_base;
    int n_tiles;
};

// Iterates the (sequence, kc-tile) work of a row tile identically in every role.
struct SegIter {
    const int32_t *cu_q, *cu_k, *cu_blocks;
    int batch, r;
    int64_t m0, m1;
    int s;
    int64_t min_bt;  // segments whose last row has b_t <= min_bt are skipped (sample mode)
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
            seg.q0 = q0;
            seg.kc_base = cu_blocks[cs];
            const int64_t t_last = (Lk - Lq) + (e - 1 - q0);
            const int64_t bt_max = t_last >= 0 ? t_last / r : 0;
            seg.n_tiles = (int)((bt_max + kBM - 1) / kBM);
            if (seg.n_tiles == 0 || bt_max <= min_bt) continue;
            return true;
        }
        return false;
    }
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); }

// What the epilogue does with the scores (IdxMode):
//   kScores  S[t, b] into the score rows (b < b_t)
//   kSample  only every stride-th kc tile is computed; its scores go to a compact
//            sample row (tile n lands at (n / stride) * 128), rows whose b_t is at
//            most min_bt are skipped
//   kEmit    every tile; (S, b) is appended to the row's candidate list when
//            S >= theta of the row (a lower bound on the row's (k-1)-th best score)
enum IdxMode { kScores = 0, kSample = 1, kEmit = 2 };

template <int kMode>
__global__ void __launch_bounds__(kIdxThreads, 1)
index_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
                const float *__restrict__ w, const int32_t *__restrict__ cu_q,
                const int32_t *__restrict__ cu_k, const int32_t *__restrict__ cu_blocks, int batch,
                int64_t row_begin, int64_t row_end, const __grid_constant__ IdxOut out, int r)
{
    const int step = kMode == kSample ? out.stride : 1;           // kc tiles advanced per iteration
    const int64_t min_bt = kMode == kSample ? out.min_bt : -1;
    float *const scores = kMode == kScores ? out.scores : out.sample;
    const int64_t ld = kMode == kScores ? out.ld : out.sample_ld;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = smem + kQBytes;
    IdxShared *sh = reinterpret_cast<IdxShared *>(sK + kStages * kKcBytes);

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
        mbar_init(&sh->q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->acc_full[i], 1);
            mbar_init(&sh->acc_empty[i], kEpiWarps);
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

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (elect_one()) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_kc);
            mbar_arrive_expect_tx(&sh->q_full, kQBytes);
            for (int c = 0; c < 2; ++c) tma_load_2d(sQ + c * kChunkQ, &map_q, &sh->q_full, c * 64, (int32_t)(m0 * 4));
            SegIter it{cu_q, cu_k, cu_blocks, batch, r, m0, m1, s0, min_bt};
            Segment seg;
            uint32_t k = 0;
            bool ok = true;
            while (ok && it.next(seg)) {
                for (int n = 0; n < seg.n_tiles; n += step, ++k) {
                    const uint32_t st = k % kStages, round = k / kStages;
                    if (!mbar_wait(&sh->empty[st], (round & 1) ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&sh->full[st], kKcBytes);
                    const int32_t y = (int32_t)(seg.kc_base + (int64_t)n * kBM);
                    for (int c = 0; c < 4; ++c)  // hi dims 0..63, 64..127, then lo
                        tma_load_2d(sK + st * kKcBytes + c * kChunkKc, &map_kc, &sh->full[st], c * 64, y);
                }
            }
            // drain: every copy issued must land before the CTA exits
            mbar_wait(&sh->q_full, 0, nullptr);
            if (!ok) {
                for (uint32_t j = (k > kStages ? k - kStages : 0); j < k; ++j)
                    mbar_wait(&sh->full[j % kStages], (j / kStages) & 1, nullptr);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kQRowsT, 0, 0);
            const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK);
            bool ok = mbar_wait(&sh->q_full, 0, abort_flag);
            SegIter it{cu_q, cu_k, cu_blocks, batch, r, m0, m1, s0, min_bt};
            Segment seg;
            uint32_t k = 0;
            while (ok && it.next(seg)) {
                for (int n = 0; n < seg.n_tiles; n += step, ++k) {
                    const uint32_t st = k % kStages, round = k / kStages;
                    const uint32_t acc = k & 1, use = k >> 1;
                    if (!mbar_wait(&sh->acc_empty[acc], (use & 1) ^ 1, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(&sh->full[st], round & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem + acc * kQRowsT;
#pragma unroll
                    for (int ks = 0; ks < 2 * kIdxDim / 16; ++ks) {  // hi plane, then lo plane
                        const int kk = ks & 7;                       // k-step within the 128 dims
                        const uint32_t koff = (kk & 3) * 32;
                        const uint64_t ad = sdesc_sw128(k_addr + st * kKcBytes + (ks >> 2) * kChunkKc + koff, 16, 1024);
                        const uint64_t bd = sdesc_sw128(q_addr + (kk >> 2) * kChunkQ + koff, 16, 1024);
                        mma_bf16_ss(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&sh->empty[st]);
                    mma_commit(&sh->acc_full[acc]);
                }
            }
        }
    } else {
        // ---------------- the epilogue (warps 2..17) ----------------
        const int et = threadIdx.x - 64;            // 0 .. 511
        if (et < kQRowsT) {  // the tile's weights, (row, head) in q_idx order
            const int64_t i = m0 + (et >> 2);
            const int row = et >> 2, h = et & 3;
            sh->wq[(row >> 1) * 8 + (h >> 1) * 4 + (h & 1) * 2 + (row & 1)] = i < m1 ? __ldg(w + i * 4 + h) : 0.f;
        }
        if (kMode == kEmit && et < kTokTile) {
            const int64_t i = m0 + et;
            sh->theta[et] = i < m1 ? __ldg(out.theta + (i - row_begin)) : INFINITY;
        }
        epi_bar();  // the weight table is complete
        // emit mode: list segment (row, quad) belongs to exactly one warp, which keeps its
        // 16 rows' lengths in its own shared-memory slots (read by every lane, advanced
        // by lane 0, ordered by the warp barrier at the end of each tile): no atomics
        int *seg_len = sh->seg_len[warp - 2];
        if (kMode == kEmit && lane < 16) seg_len[lane] = 0;
        __syncwarp();
        const int cap_q = out.list_cap / 4;

        const int ew = warp - 2;
        const int quad = warp & 3;                 // TMEM lane quadrant this warp may read
        const int part = ew >> 2;                  // rows [16 part, 16 part + 16) of the tile
        const int b_local = quad * 32 + lane;      // kc block within the tile (TMEM lane)
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float4 *wq4 = reinterpret_cast<const float4 *>(sh->wq);

        SegIter it{cu_q, cu_k, cu_blocks, batch, r, m0, m1, s0, min_bt};
        Segment seg;
        uint32_t k = 0;
        bool ok = true;
        const uint32_t lt_mask = (1u << lane) - 1u;
        while (ok && it.next(seg)) {
            // this thread's rows j (bit j of vmask) belong to the segment; row j sits at
            // t = t0 + j, b_t = t >> rs (r a power of two); blocks b < b_t are scored
            const int64_t i0 = m0 + part * 16;
            const int j_lo = (int)(seg.seg_begin > i0 ? (seg.seg_begin - i0 < 16 ? seg.seg_begin - i0 : 16) : 0);
            const int j_hi = (int)(seg.seg_end > i0 ? (seg.seg_end - i0 < 16 ? seg.seg_end - i0 : 16) : 0);
            const uint32_t vmask = j_hi > j_lo ? (((1u << j_hi) - 1u) & ~((1u << j_lo) - 1u)) : 0u;
            const int32_t t0 = (int32_t)(seg.pos_offset + (i0 - seg.q0));
            const int rs = 31 - __clz(r);
            if (kMode == kScores && j_hi > j_lo && ((t0 + j_hi - 1) >> rs) > ld) set_device_status(QSA_ERR_DEVICE_CHECK);
            const int32_t cap = ld < 0x7FFFFFFF ? (int32_t)ld : 0x7FFFFFFF;  // score / sample columns
            float *row0 = kMode == kEmit ? nullptr : scores + (i0 - row_begin) * ld;
            // emit mode: segment (row i0 + j, quad) starts at lbase + j * 4 cap_q
            uint2 *const lbase = kMode == kEmit ? out.lists + ((i0 - row_begin) * 4 + quad) * cap_q : nullptr;
            for (int n = 0; n < seg.n_tiles; n += step, ++k) {
                const uint32_t acc = k & 1, use = k >> 1;
                if (!mbar_wait(&sh->acc_full[acc], use & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const int32_t b = n * kBM + b_local;
                const int32_t col = kMode == kSample ? (n / step) * kBM + b_local : b;  // where the score goes
                const bool col_ok = kMode == kEmit || col < cap;
                // warp-uniform: all 16 rows belong to the segment and see every block of the tile
                const bool full = vmask == 0xFFFFu && n * kBM + kBM <= (t0 >> rs);
                float *p = row0 + col;
                const uint32_t tbase = tmem + lane_addr + acc * kQRowsT + part * 64;
                // one tile of this thread (kc block b, 16 rows): the whole-tile case is compiled
                // apart, without the per-row causal test
                auto tile = [&](auto full_tag) {
                    constexpr bool kFull = decltype(full_tag)::value;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float v[16];  // rows 16 part + 4 c .. + 3, heads 0..3
                        tmem_ld16(tbase + c * 16, v);
                        tmem_wait_ld();
                        // the 4 rows' scores, two rows per packed fp32x2 operation (each lane of
                        // an fp32x2 op rounds as the scalar op does: the same bits)
                        float sc[4];
#pragma unroll
                        for (int jp = 0; jp < 4; jp += 2) {
                            const int pr = part * 8 + c * 2 + jp / 2;  // row pair of the tile
                            const float4 w01 = wq4[2 * pr], w23 = wq4[2 * pr + 1];
                            const float *va = v + 4 * jp, *vb = v + 4 * jp + 4;
                            float2 x = __fmul2_rn(make_float2(w01.x, w01.y),
                                                  make_float2(fmaxf(va[0], 0.f), fmaxf(vb[0], 0.f)));
                            x = __ffma2_rn(make_float2(w01.z, w01.w), make_float2(fmaxf(va[1], 0.f), fmaxf(vb[1], 0.f)), x);
                            x = __ffma2_rn(make_float2(w23.x, w23.y), make_float2(fmaxf(va[2], 0.f), fmaxf(vb[2], 0.f)), x);
                            x = __ffma2_rn(make_float2(w23.z, w23.w), make_float2(fmaxf(va[3], 0.f), fmaxf(vb[3], 0.f)), x);
                            sc[jp] = x.x;
                            sc[jp + 1] = x.y;
                        }
                        if (kMode != kEmit) {
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const int j = c * 4 + jj;
                                const bool in = kFull ? col_ok : (((vmask >> j) & 1u) && b < ((t0 + j) >> rs) && col_ok);
                                if (in) __stcs(p, sc[jj]);
                                p += ld;
                            }
                        } else {
                            // append (S, b) to this warp's segment of row j's list when S >= theta:
                            // the warp's hits take consecutive slots in ballot order
                            const float4 th4 = reinterpret_cast<const float4 *>(sh->theta)[part * 4 + c];
                            const float th[4] = {th4.x, th4.y, th4.z, th4.w};
                            uint32_t m[4], any = 0u;
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const int j = c * 4 + jj;
                                const bool in = kFull || (((vmask >> j) & 1u) && b < ((t0 + j) >> rs));
                                m[jj] = __ballot_sync(0xffffffffu, in && sc[jj] >= th[jj]);
                                any |= m[jj];
                            }
                            if (any != 0u) {  // warp-uniform
#pragma unroll
                                for (int jj = 0; jj < 4; ++jj) {
                                    if (m[jj] == 0u) continue;  // warp-uniform
                                    const int j = c * 4 + jj;
                                    const int len = seg_len[j];
                                    const int pos = len + __popc(m[jj] & lt_mask);
                                    if (((m[jj] >> lane) & 1u) && pos < cap_q)
                                        lbase[j * 4 * cap_q + pos] = make_uint2(__float_as_uint(sc[jj]), (uint32_t)b);
                                    if (lane == 0) seg_len[j] = len + __popc(m[jj]);  // read again only after
                                }                                                      // the tile's warp barrier
                            }
                        }
                    }
                };
                if (full)
                    tile(std::true_type{});
                else
                    tile(std::false_type{});
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh->acc_empty[acc]);
            }
        }
        if (kMode == kEmit) {  // the lengths of this warp's 16 list segments (lane j: row j)
            __syncwarp();
            const int mine = lane < 16 ? seg_len[lane] : 0;
            const int64_t i = m0 + part * 16 + lane;
            if (lane < 16 && i < m1) out.counts[(i - row_begin) * 4 + quad] = mine;
        }
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

// kPlanes = 2: the exact scores (hi + lo planes); 1: the hi plane only (the decode
// selector then refines the near-threshold blocks exactly)
template <int kPlanes>
__global__ void __launch_bounds__(kRowWarps * 32)
index_rowwise_kernel(const __nv_bfloat16 *__restrict__ q_idx, const float *__restrict__ w,
                     const __nv_bfloat16 *__restrict__ kc, const int32_t *__restrict__ cu_q,
                     const int32_t *__restrict__ cu_k, const int32_t *__restrict__ cu_blocks,
                     int batch, int64_t row_begin, float *__restrict__ scores, int64_t ld, int r)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t i = row_begin + blockIdx.y;
    // cu_q == nullptr: decode rows, row i is sequence i at t = L - 1
    const int s = cu_q != nullptr ? find_seq(cu_q, batch, i) : (int)i;
    const int64_t Lk = (int64_t)cu_k[s + 1] - cu_k[s];
    const int64_t Lq = cu_q != nullptr ? (int64_t)cu_q[s + 1] - cu_q[s] : 1;
    const int64_t t = cu_q != nullptr ? (Lk - Lq) + (i - cu_q[s]) : Lk - 1;
    int64_t bt = t >= 0 ? t / r : 0;
    if (bt > ld || (int64_t)cu_blocks[s + 1] - cu_blocks[s] != Lk / r) {
        if (threadIdx.x == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        if ((int64_t)cu_blocks[s + 1] - cu_blocks[s] != Lk / r) return;
        bt = ld;
    }
    const int64_t c0 = (int64_t)blockIdx.x * kRowChunk;
    const int64_t c1 = (c0 + kRowChunk < bt) ? c0 + kRowChunk : bt;
    if (c0 >= c1) return;

    index_row_cuda<kPlanes>(q_idx + i * 512, w + i * 4, kc + (int64_t)cu_blocks[s] * 256, c0, c1,
                   scores + (int64_t)blockIdx.y * ld, warp, kRowWarps, lane);
}

// ------------------------------------------------------------------ decode GEMV on the tensor cores
// The decode scan of the hi planes as a stream of TMA tiles: per 128-block kc tile,
// D[b, h] = <hi_b, q_h> with the kc tile as the M = 128 side and the row's 4 heads
// (plus 12 zero rows) as the N = 16 side, 8 MMAs of K = 16; an epilogue thread per
// block (TMEM lane) sums w_h ReLU(D[b, h]) and stores a coalesced score row.  The
// tensor cores take the arithmetic off the CUDA cores, so the kernel streams the
// hi planes at the HBM rate.
constexpr int kGvBN = 16;                       // N: 4 heads + 12 zero rows
constexpr int kGvChunkQ = kGvBN * 128;          // 2 KB: one 64-dim chunk of the q tile
constexpr int kGvTile = 128 * 128 * 2;          // 32 KB: a 128-block tile of hi planes
constexpr int kGvStages = 3;
constexpr int kGvChunk = 1024;                  // kc blocks per CTA (8 tiles)
constexpr int kGvThreads = 192;
constexpr int kGvSmem = 2 * kGvChunkQ + kGvStages * kGvTile + 256 + 1024;

__global__ void __launch_bounds__(kGvThreads, 2)
index_gemv_hi_kernel(const __grid_constant__ CUtensorMap map_kc, const __nv_bfloat16 *__restrict__ q_idx,
                     const float *__restrict__ w, const int32_t *__restrict__ cu_q,
                     const int32_t *__restrict__ cu_k, const int32_t *__restrict__ cu_blocks, int batch,
                     int64_t row_begin, float *__restrict__ scores, int64_t ld, int r)
{
    pdl_enter();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem;                               // stages of kc tiles (1 KB aligned)
    uint8_t *sQ = smem + kGvStages * kGvTile;         // the q tile
    uint64_t *full = reinterpret_cast<uint64_t *>(sQ + 2 * kGvChunkQ);
    uint64_t *empty = full + kGvStages;
    uint64_t *acc_full = empty + kGvStages;           // [2]
    uint64_t *acc_empty = acc_full + 2;               // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    int *abort_slot = reinterpret_cast<int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int64_t i = row_begin + blockIdx.y;
    const int s = cu_q != nullptr ? find_seq(cu_q, batch, i) : (int)i;
    const int64_t Lk = (int64_t)cu_k[s + 1] - cu_k[s];
    const int64_t Lq = cu_q != nullptr ? (int64_t)cu_q[s + 1] - cu_q[s] : 1;
    const int64_t t = cu_q != nullptr ? (Lk - Lq) + (i - cu_q[s]) : Lk - 1;
    int64_t bt = t >= 0 ? t / r : 0;
    if (bt > ld) {
        if (threadIdx.x == 0) set_device_status(QSA_ERR_DEVICE_CHECK);
        bt = ld;
    }
    const int64_t c0 = (int64_t)blockIdx.x * kGvChunk;
    const int64_t c1 = (c0 + kGvChunk < bt) ? c0 + kGvChunk : bt;
    if (c0 >= c1) return;  // uniform: the whole CTA leaves before any set-up
    const int n_tiles = (int)((c1 - c0 + 127) / 128);
    const int64_t kc0 = (int64_t)cu_blocks[s] + c0;

    // the q tile: rows 0..3 the row's 4 heads, rows 4..15 zero (128-byte swizzle, K-major)
    for (int x = threadIdx.x; x < 2 * kGvChunkQ / 16; x += kGvThreads) {
        const int ch = x / (kGvChunkQ / 16), row = (x % (kGvChunkQ / 16)) / 8, u = x % 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < 4) v = *reinterpret_cast<const uint4 *>(q_idx + (i * 4 + row) * 128 + ch * 64 + u * 8);
        *reinterpret_cast<uint4 *>(sQ + ch * kGvChunkQ + row * 128 + ((u ^ (row & 7)) << 4)) = v;
    }
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        for (int x = 0; x < kGvStages; ++x) {
            mbar_init(&full[x], 1);
            mbar_init(&empty[x], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&acc_full[x], 1);
            mbar_init(&acc_empty[x], 4);
        }
        *abort_slot = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int *abort_flag = abort_slot;

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&map_kc);
            int n = 0;
#ifdef QSA_DEBUG_CHECKS
            const bool skip_tile1 = g_debug_fault_site == 1;
#endif
            for (; n < n_tiles; ++n) {
                const uint32_t st = n % kGvStages, round = n / kGvStages;
                if (!mbar_wait(&empty[st], (round & 1) ^ 1, abort_flag)) break;
#ifdef QSA_DEBUG_CHECKS
                if (skip_tile1 && n == 1) continue;  // injected fault: tile 1's full barrier never completes
#endif
                mbar_arrive_expect_tx(&full[st], kGvTile);
                for (int c = 0; c < 2; ++c)  // the hi plane: dims 0..63, 64..127
                    tma_load_2d(sK + st * kGvTile + c * (kGvTile / 2), &map_kc, &full[st], c * 64,
                                (int32_t)(kc0 + (int64_t)n * 128));
            }
            if (n < n_tiles)  // gave up: the copies in flight land before the CTA exits
                for (int j = (n > kGvStages ? n - kGvStages : 0); j < n; ++j)
                    mbar_wait(&full[j % kGvStages], (j / kGvStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, kGvBN, 0, 0);
            const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK);
            for (int n = 0; n < n_tiles; ++n) {
                const uint32_t st = n % kGvStages, round = n / kGvStages;
                const uint32_t acc = n & 1, use = n >> 1;
                if (!mbar_wait(&acc_empty[acc], (use & 1) ^ 1, abort_flag)) break;
                if (!mbar_wait(&full[st], round & 1, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t koff = (ks & 3) * 32;
                    const uint64_t ad = sdesc_sw128(k_addr + st * kGvTile + (ks >> 2) * (kGvTile / 2) + koff, 16, 1024);
                    const uint64_t bd = sdesc_sw128(q_addr + (ks >> 2) * kGvChunkQ + koff, 16, 1024);
                    mma_bf16_ss(tmem + acc * kGvBN, ad, bd, idesc, ks > 0 ? 1u : 0u);
                }
                mma_commit(&empty[st]);
                mma_commit(&acc_full[acc]);
            }
        }
    } else {
        const int quad = warp & 3;
        const int b_local = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float4 wv = *reinterpret_cast<const float4 *>(w + i * 4);
        float *srow = scores + (int64_t)blockIdx.y * ld;
        for (int n = 0; n < n_tiles; ++n) {
            const uint32_t acc = n & 1, use = n >> 1;
            if (!mbar_wait(&acc_full[acc], use & 1, abort_flag)) break;
            tc_fence_after();
            float v[8];
            tmem_ld8(tmem + lane_addr + acc * kGvBN, v);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            float sc = wv.x * fmaxf(v[0], 0.f);
            sc = fmaf(wv.y, fmaxf(v[1], 0.f), sc);
            sc = fmaf(wv.z, fmaxf(v[2], 0.f), sc);
            sc = fmaf(wv.w, fmaxf(v[3], 0.f), sc);
            const int64_t b = c0 + (int64_t)n * 128 + b_local;
            if (b < c1) srow[b] = sc;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 32);
    }
}

}  // namespace

cudaError_t launch_index_tc_mode(const IndexArgs &a, const IdxOut &out, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0 || a.kc_rows <= 0) return cudaSuccess;
    CUtensorMap mq, mk;
    // q_idx as [total_q * 4, 128] bf16, 256-row boxes; kc as [kc_rows, 256] bf16 (hi plane, then
    // lo plane), boxes of 64 columns x 128 rows
    if (!make_tmap_2d(&mq, a.q_idx, 128, (uint64_t)a.total_q * 4, 256, 64, kQRowsT)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&mk, a.kc, 256, (uint64_t)a.kc_rows, 512, 64, kBM)) return cudaErrorInvalidValue;
    if (out.mode == kSample && out.stride <= 0) return cudaErrorInvalidValue;
    auto kern = out.mode == kSample ? index_tc_kernel<kSample>
                                    : (out.mode == kEmit ? index_tc_kernel<kEmit> : index_tc_kernel<kScores>);
    {
        const cudaError_t e = set_smem_attr_once(reinterpret_cast<const void *>(kern), kIdxSmem);
        if (e != cudaSuccess) return e;
    }
    const int64_t tiles = (rows + kTokTile - 1) / kTokTile;
    kern<<<(unsigned)tiles, kIdxThreads, kIdxSmem, stream>>>(mq, mk, a.w, a.cu_q, a.cu_k, a.cu_blocks, a.batch,
                                                             a.row_begin, a.row_end, out, a.r);
    return cudaGetLastError();
}

cudaError_t launch_index_tc(const IndexArgs &a, cudaStream_t stream)
{
    IdxOut out{};
    out.mode = kScores;
    out.scores = a.scores;
    out.ld = a.ld;
    return launch_index_tc_mode(a, out, stream);
}

template <int kPlanes>
static cudaError_t launch_rowwise(const IndexArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0 || a.kc_rows <= 0) return cudaSuccess;
    const int64_t chunks = (a.ld + kRowChunk - 1) / kRowChunk;
    for (int64_t done = 0; done < rows; done += 65535) {
        const int64_t n = rows - done < 65535 ? rows - done : 65535;
        dim3 grid((unsigned)chunks, (unsigned)n);
        index_rowwise_kernel<kPlanes><<<grid, kRowWarps * 32, 0, stream>>>(
            a.q_idx, a.w, a.kc, a.cu_q, a.cu_k, a.cu_blocks, a.batch, a.row_begin + done,
            a.scores + done * a.ld, a.ld, a.r);
    }
    return cudaGetLastError();
}

cudaError_t launch_index_rowwise(const IndexArgs &a, cudaStream_t stream) { return launch_rowwise<2>(a, stream); }

cudaError_t launch_index_rowwise_hi(const IndexArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0 || a.kc_rows <= 0) return cudaSuccess;
    // w rows are read as float4: 16-byte aligned (the caller's fp32 [rows, 4] array)
    // (and kc tile rows are int32 TMA coordinates)
    if ((reinterpret_cast<uintptr_t>(a.w) & 15u) != 0 || a.kc_rows > (int64_t)INT32_MAX - 2 * kGvChunk)
        return launch_rowwise<1>(a, stream);
    CUtensorMap mk;
    if (!make_tmap_2d(&mk, a.kc, 256, (uint64_t)a.kc_rows, 512, 64, 128)) return cudaErrorInvalidValue;
    {
        const cudaError_t e = set_smem_attr_once(reinterpret_cast<const void *>(index_gemv_hi_kernel), kGvSmem);
        if (e != cudaSuccess) return e;
    }
    const int64_t chunks = (a.ld + kGvChunk - 1) / kGvChunk;
    for (int64_t done = 0; done < rows; done += 65535) {
        const int64_t n = rows - done < 65535 ? rows - done : 65535;
        const cudaError_t e = launch_pdl(index_gemv_hi_kernel, dim3((unsigned)chunks, (unsigned)n), dim3(kGvThreads),
                                         kGvSmem, stream, mk, a.q_idx, a.w, a.cu_q, a.cu_k, a.cu_blocks, a.batch,
                                         a.row_begin + done, a.scores + done * a.ld, a.ld, a.r);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace qsa
