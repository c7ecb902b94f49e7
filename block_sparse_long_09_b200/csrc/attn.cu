// attn.cu -- QSA sparse GQA core attention (prefill and split-K decode).
//
// "On the Design of Qwen3.8 Next Architecture" (reading notes), section 6: the
// selected micro-blocks are expanded to their token indices and handed to the
// sparse core attention, O(nK) for a fixed budget K = 2048 tokens.  Heads per
// the "Model Summary" table: 24 query heads, 2 KV heads (12 query heads per
// group), head dim 256.  Query t sees the tokens of its selected blocks with
// j <= t (causal inside its own block).
//
// The kernel is bound by the gather: 4 MiB of K/V per query, scattered in
// 4 KB micro-blocks, against ~25 MFLOP of math.  Design (B200):
//  * One TMA op per micro-block and tensor: a 3-D tensor map over K (or V)
//    with dims (64 d, token-row, 4 d-chunks) and strides (512 B, 128 B) copies
//    the block's 8 rows (4 tokens x 2 KV heads) x 256 d = 4 KB straight into
//    the 128-byte-swizzled K-major UMMA layout (8-row atom per block, SBO 4 KB).
//    Fewer, larger TMA ops is what lifts the gather rate: 512 B boxes stall at
//    ~2.4 TB/s on B200, whole blocks stream at the HBM rate.
//  * Both KV groups ride in one MMA: rows alternate (token, group), so
//    S^T[128 rows, 32] = K_tile . Q^T carries all 24 heads (8 pad); entries
//    whose head belongs to the other group are masked, and P^T keeps them at
//    zero, so O^T[256 d, 32] += V_tile^T . P^T accumulates every head at once.
//    Keys are the M = 128 side ("swap AB"): the tensor cores idle anyway.
//  * Online softmax, lazy rescale: the running max is updated per 64-token
//    tile (exact per-head tile max, one named barrier), O is rescaled in TMEM
//    only when a new max exceeds the old by more than 2^8 in probability.
//  * Warp roles of a persistent CTA (one per SM):
//      warp 0      TMA producer: Q (per item), then K/V tiles in MMA order
//                  (K0, K1, V0, K2, V1, ...) through a 3-slot ring of 64 KB;
//                  block ids are loaded three tiles ahead (across items) and
//                  checked at use, so their latency stays off the issue path
//      warp 1      TMEM owner + single-thread tcgen05.mma issue: S(j+1) is
//                  issued before PV(j) so QK^T overlaps the softmax
//      warps 2..5  softmax (thread = TMEM lane = (token, group) row) and the
//                  epilogue (thread = d); split-K decode writes fp32 partial
//                  states that combine_kernel merges.
// Without a selection array the kernel attends to every block j <= t: that is
// the dense flash-decoding baseline (one query per sequence, split-K).
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kHQ = 24, kHKV = 2, kD = 256, kGrp = kHQ / kHKV;
constexpr int kBlkTile = 16;                    // micro-blocks per tile (r = 4)
constexpr int kRowsTile = 128;                  // 16 blocks x 4 tokens x 2 KV heads
constexpr int kBlockBytes = 8 * kD * 2;         // 4 KB: one block of K (or V), both heads
constexpr int kSlotBytes = kBlkTile * kBlockBytes;  // 64 KB
constexpr int kNSlot = 3;
constexpr int kQRows = 32;                      // 24 heads + 8 pad
constexpr int kQChunk = kQRows * 128;           // 4 KB: 64 d-columns of Q
constexpr int kQBytes = 4 * kQChunk;            // 16 KB
constexpr int kPChunk = kQRows * 128;           // 4 KB: P^T, 32 heads x 64 rows
constexpr int kPBytes = 2 * kPChunk;            // 8 KB: 32 heads x 128 rows
constexpr int kNP = 2;
constexpr int kAttThreads = 192;
constexpr uint32_t kSCol = 0, kOCol = 64, kTmemCols = 128;  // S: 2 x 32 cols, O^T: 2 halves x 32
constexpr float kRescaleLog2 = 8.f;             // lazy-rescale threshold (probability 2^8)

struct AttShared {
    uint64_t slot_full[kNSlot], slot_empty[kNSlot];
    uint64_t q_full, q_empty;
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[kNP], p_empty[kNP];
    uint64_t o_full;               // once per item: every PV of the item has completed
    uint64_t sc_full[2], sc_empty[2];  // decode kernel: a chunk's S in TMEM is complete / consumed
    uint32_t tmem_base;
    int abort_flag;
    int64_t ev_ts, ev_te, ev_r0s;  // even schedule: this CTA's tiles [ts, te); first tile of row r0
    int ev_r0, ev_nseg;            // first row and number of rows it touches
    float red_max[2][4][2][kGrp];  // [tile parity][quad][group][head]
    float red_sum[4][2][kGrp];
};

constexpr int kOffQ = kNSlot * kSlotBytes;
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kOffShared = kOffP + kNP * kPBytes;
constexpr int kAttSmem = kOffShared + (int)sizeof(AttShared) + 1024;
static_assert(kAttSmem <= 232448, "shared memory of one CTA");

struct RowInfo {
    int64_t row;    // packed query row
    int64_t rl;     // row within the call (row - row_begin)
    int s;
    int sp;         // split (or key chunk) of this item
    int64_t t, bt, tok_base;
    int nsel;       // valid selection slots of the row
    int p0, p1;     // selection positions [p0, p1) handled by this item
    int nt;         // 16-block tiles covering [p0, p1)
    int64_t slot;   // partial-state slot (schedules that merge partial states)
};

// Work item -> (row, selection range).  Three schedules:
//  * nsplit == 1: one item per row, the whole selection;
//  * split-K (bounds == nullptr, nsplit > 1): item = rl * nsplit + sp, split sp takes
//    tiles [sp * tps, (sp + 1) * tps) of the row's selection;
//  * key-chunked (bounds != nullptr): item = sp * rows + rl (chunk-major, so all CTAs
//    gather from the same L2-resident key chunk sp); the range comes from bounds.
__device__ __forceinline__ RowInfo row_info(int64_t item, int nsplit, int64_t rows, int64_t row_begin,
                                            const int32_t *cu_q, const int32_t *cu_k, int batch,
                                            int kb, int r, const int32_t *bounds)
{
    RowInfo ri;
    if (bounds != nullptr) {
        ri.rl = item % rows;
        ri.sp = (int)(item / rows);
    } else {
        ri.rl = item / nsplit;
        ri.sp = (int)(item % nsplit);
    }
    ri.row = row_begin + ri.rl;
    if (cu_q != nullptr) {
        ri.s = find_seq(cu_q, batch, ri.row);
        const int64_t Lq = (int64_t)cu_q[ri.s + 1] - cu_q[ri.s];
        const int64_t Lk = (int64_t)cu_k[ri.s + 1] - cu_k[ri.s];
        ri.t = (Lk - Lq) + (ri.row - cu_q[ri.s]);
    } else {
        ri.s = (int)ri.row;
        ri.t = (int64_t)cu_k[ri.s + 1] - cu_k[ri.s] - 1;
    }
    const bool ok = ri.t >= 0;
    ri.bt = ok ? ri.t / r : 0;
    ri.tok_base = cu_k[ri.s];
    const int64_t nsel = ri.bt + 1 < kb ? ri.bt + 1 : kb;
    ri.nsel = (int)nsel;
    if (bounds != nullptr) {
        ri.p0 = bounds[ri.rl * (nsplit + 1) + ri.sp];
        ri.p1 = bounds[ri.rl * (nsplit + 1) + ri.sp + 1];
        if (ri.p1 > ri.nsel) ri.p1 = ri.nsel;
    } else {
        const int max_tiles = (kb + kBlkTile - 1) / kBlkTile;
        const int tps = (max_tiles + nsplit - 1) / nsplit;
        ri.p0 = ri.sp * tps * kBlkTile;
        const int e = (ri.sp + 1) * tps * kBlkTile;
        ri.p1 = e < ri.nsel ? e : ri.nsel;
    }
    if (!ok || ri.p0 < 0 || ri.p1 < ri.p0) ri.p1 = ri.p0 = 0;
    ri.nt = (ri.p1 - ri.p0 + kBlkTile - 1) / kBlkTile;
    ri.slot = ri.rl * nsplit + ri.sp;
    return ri;
}

// Even schedule (decode): the batch's (row, tile) units in row order, cut into
// gridDim.x equal shares, share c = tiles [c T / G, (c + 1) T / G).  A row cut by a
// share boundary is attended in pieces whose softmax states a second kernel merges:
// the piece at the row's first tile writes slot G + row, a piece that starts inside
// the row (always the first piece of a share) writes slot c.

// tiles of decode row s (one query at t = L_s - 1); 0 for an empty sequence
__device__ __forceinline__ int decode_tiles(const int32_t *cu_k, int64_t s, int kb, int r)
{
    const int64_t t = (int64_t)__ldg(cu_k + s + 1) - __ldg(cu_k + s) - 1;
    if (t < 0) return 0;
    const int64_t nsel = t / r + 1 < kb ? t / r + 1 : kb;
    return (int)((nsel + kBlkTile - 1) / kBlkTile);
}

// one warp: this CTA's share [ts, te), the rows it touches, the first tile of the first;
// CTA 0 also stores every row's first tile (and the total) for the merge kernel
__device__ __forceinline__ void even_setup(AttShared *sh, const int32_t *cu_k, int64_t row_begin, int64_t rows,
                                           int kb, int r, int lane, int64_t *tile_prefix)
{
    if (blockIdx.x == 0) {
        int64_t acc = 0;
        for (int64_t base = 0; base < rows; base += 32) {
            const int64_t i = base + lane;
            const int nt = i < rows ? decode_tiles(cu_k, row_begin + i, kb, r) : 0;
            int incl = nt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            if (i < rows) tile_prefix[i] = acc + incl - nt;
            acc += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) tile_prefix[rows] = acc;
    }
    int64_t total = 0;
    for (int64_t base = 0; base < rows; base += 32) {
        const int64_t i = base + lane;
        total += __reduce_add_sync(0xffffffffu, i < rows ? decode_tiles(cu_k, row_begin + i, kb, r) : 0);
    }
    const int64_t grid = gridDim.x;
    const int64_t ts = (int64_t)blockIdx.x * total / grid, te = ((int64_t)blockIdx.x + 1) * total / grid;
    // r0: the first row whose tiles end after ts; r1: the first row whose tiles reach te
    int64_t acc = 0, r0 = 0, r0s = 0, r1 = 0;
    bool f0 = false, f1 = false;
    for (int64_t base = 0; base < rows && !(f0 && f1); base += 32) {
        const int64_t i = base + lane;
        const int nt = i < rows ? decode_tiles(cu_k, row_begin + i, kb, r) : 0;
        int incl = nt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const int64_t st = acc + incl - nt, en = acc + incl;
        const uint32_t h0 = __ballot_sync(0xffffffffu, nt > 0 && en > ts);
        const uint32_t h1 = __ballot_sync(0xffffffffu, nt > 0 && en >= te);
        if (!f0 && h0 != 0u) {  // warp-uniform
            const int l = __ffs(h0) - 1;
            r0 = base + l;
            r0s = __shfl_sync(0xffffffffu, st, l);
            f0 = true;
        }
        if (!f1 && h1 != 0u) {
            r1 = base + __ffs(h1) - 1;
            f1 = true;
        }
        acc += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        sh->ev_ts = ts;
        sh->ev_te = te;
        sh->ev_r0 = (int)r0;
        sh->ev_r0s = r0s;
        sh->ev_nseg = (te > ts && f0 && f1) ? (int)(r1 - r0 + 1) : 0;
    }
}

// item j of this CTA under the even schedule: row r0 + j cut to the share
__device__ __forceinline__ RowInfo row_info_even(int64_t j, const AttShared *sh, const int32_t *cu_k,
                                                 int64_t row_begin, int kb, int r)
{
    RowInfo ri;
    int64_t rs = sh->ev_r0s;  // first tile of the row
    for (int64_t q = 0; q < j; ++q) rs += decode_tiles(cu_k, row_begin + sh->ev_r0 + q, kb, r);
    ri.rl = sh->ev_r0 + j;
    ri.row = row_begin + ri.rl;
    ri.s = (int)ri.row;
    ri.sp = 0;
    ri.t = (int64_t)__ldg(cu_k + ri.s + 1) - __ldg(cu_k + ri.s) - 1;
    const bool ok = ri.t >= 0;
    ri.bt = ok ? ri.t / r : 0;
    ri.tok_base = __ldg(cu_k + ri.s);
    ri.nsel = (int)(ri.bt + 1 < kb ? ri.bt + 1 : kb);
    const int ntr = ok ? (ri.nsel + kBlkTile - 1) / kBlkTile : 0;
    const int64_t a = sh->ev_ts > rs ? sh->ev_ts : rs;
    const int64_t b = sh->ev_te < rs + ntr ? sh->ev_te : rs + ntr;
    if (b <= a) {
        ri.p0 = ri.p1 = ri.nt = 0;
        ri.slot = 0;
        return ri;
    }
    ri.p0 = (int)((a - rs) * kBlkTile);
    const int e = (int)((b - rs) * kBlkTile);
    ri.p1 = e < ri.nsel ? e : ri.nsel;
    ri.nt = (int)(b - a);
    ri.slot = a == rs ? (int64_t)gridDim.x + ri.rl : (int64_t)blockIdx.x;
    return ri;
}

constexpr int32_t kNoBlock = INT32_MIN;  // a position past the item's selection range

// raw block id at selection position pos of an item, unchecked (so that the load's
// latency is paid only where the id is used): kNoBlock outside [p0, p1); without a
// selection (sel == nullptr, dense attention) position pos is block pos
__device__ __forceinline__ int32_t load_block(const int32_t *sel, const RowInfo &ri, int kb, int pos)
{
    if (pos >= ri.p1) return kNoBlock;
    if (sel == nullptr) return pos;
    return __ldg(sel + ri.row * kb + pos);
}

// the id to gather, or -1 (nothing: past the range, or an id outside 0 .. b_t,
// which is flagged)
__device__ __forceinline__ int32_t check_block(int32_t raw, const RowInfo &ri)
{
    if (raw == kNoBlock) return -1;
    if (raw < 0 || raw > ri.bt) {
        set_device_status(QSA_ERR_DEVICE_CHECK);
        return -1;
    }
    return raw;
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// barrier of the 128 softmax threads that also ORs a predicate over them
__device__ __forceinline__ bool softmax_any(bool x)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)x)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void st_shared_b16(uint32_t addr, uint16_t v)
{
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
        " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
        " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
          "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
          "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
          "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
          "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
          "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(kAttThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const int32_t *__restrict__ sel,
                   const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k, int batch,
                   int64_t row_begin, int64_t rows, int nsplit, int kb, int r, float scale,
                   __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out,
                   float *__restrict__ ws, const int32_t *__restrict__ bounds)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sSlot = smem;
    uint8_t *sQ = smem + kOffQ;
    uint8_t *sP = smem + kOffP;
    AttShared *sh = reinterpret_cast<AttShared *>(smem + kOffShared);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNSlot; ++i) {
            mbar_init(&sh->slot_full[i], 1);
            mbar_init(&sh->slot_empty[i], 1);
        }
        mbar_init(&sh->q_full, 1);
        mbar_init(&sh->q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->s_full[i], 1);
            mbar_init(&sh->s_empty[i], 128);
        }
        for (int i = 0; i < kNP; ++i) {
            mbar_init(&sh->p_full[i], 128);
            mbar_init(&sh->p_empty[i], 1);
        }
        mbar_init(&sh->o_full, 1);
        sh->abort_flag = 0;
        fence_barrier_init();
    }
    // P^T entries of the other KV group and of the pad heads stay zero for good
    for (int i = threadIdx.x; i < kNP * kPBytes / 16; i += kAttThreads)
        reinterpret_cast<uint4 *>(sP)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    volatile int *abort_flag = &sh->abort_flag;
    // this CTA's work items, in the same order for every role
    const int64_t it_begin = blockIdx.x, it_end = rows * nsplit, it_step = gridDim.x;
    const bool partials = nsplit > 1;
    const int64_t n_slots = rows * nsplit;  // partial-state slots
    auto item_info = [&](int64_t item) -> RowInfo {
        return row_info(item, nsplit, rows, row_begin, cu_q, cu_k, batch, kb, r, bounds);
    };

    if (warp == 0) {
        // ======================= TMA producer (whole warp) =======================
        if (lane == 0) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_k);
            tma_prefetch_desc(&map_v);
        }
        uint32_t slot_it = 0, q_it = 0;
        bool ok = true;
        const uint64_t kv_policy = make_policy_evict_last();  // K/V stay in L2 while reused
        auto issue = [&](const CUtensorMap *map, const RowInfo &ri, int32_t blk) -> bool {
            const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
            bool good = true;
            if (lane == 0) {
                good = mbar_wait(&sh->slot_empty[st], (round & 1) ^ 1, abort_flag);
                if (good) mbar_arrive_expect_tx(&sh->slot_full[st], kSlotBytes);
            }
            good = __shfl_sync(0xffffffffu, good, 0);
            if (!good) return false;
            if (lane < kBlkTile) {
                // rows (token, group) of the block; padding reads an out-of-range box (zeros)
                const int32_t y = blk >= 0 ? (int32_t)((ri.tok_base + (int64_t)blk * r) * kHKV) : -8;
                tma_load_3d_hint(sSlot + st * kSlotBytes + lane * kBlockBytes, map, &sh->slot_full[st], 0, y, 0,
                                 kv_policy);
            }
            ++slot_it;
            return true;
        };
        // Block ids stream through a window w0..w3 of raw loads that runs three tiles
        // ahead of the issue point, across item boundaries (the same item order as the
        // issue loop); an id is checked only when its tile is issued.
        int64_t pf_item = it_begin;
        RowInfo pf_ri;
        pf_ri.nt = 0;
        int pf_tile = 0;
        auto pf_seek = [&]() {  // the cursor's next item with tiles, or past the end
            for (; pf_item < it_end; pf_item += it_step) {
                pf_ri = item_info(pf_item);
                if (pf_ri.nt > 0) return;
            }
        };
        auto pf_next = [&]() -> int32_t {  // this lane's raw id of the cursor's tile; advance
            int32_t v = kNoBlock;
            if (pf_item < it_end) {
                if (lane < kBlkTile) v = load_block(sel, pf_ri, kb, pf_ri.p0 + pf_tile * kBlkTile + lane);
                if (++pf_tile == pf_ri.nt) {
                    pf_tile = 0;
                    pf_item += it_step;
                    pf_seek();
                }
            }
            return v;
        };
        pf_seek();
        int32_t w0 = pf_next();
        int32_t w1 = pf_next();
        int32_t w2 = pf_next();
        for (int64_t item = it_begin; ok && item < it_end; item += it_step) {
            const RowInfo ri = item_info(item);
            if (ri.nt == 0) continue;
            if (lane == 0) {
                ok = mbar_wait(&sh->q_empty, (q_it & 1) ^ 1, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(&sh->q_full, kQBytes);
                    for (int c = 0; c < 4; ++c)
                        tma_load_2d(sQ + c * kQChunk, &map_q, &sh->q_full, c * 64, (int32_t)(ri.row * kHQ));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ++q_it;
            if (!ok) break;
            ok = issue(&map_k, ri, check_block(w0, ri));
            for (int jl = 0; ok && jl < ri.nt; ++jl) {
                const int32_t w3 = pf_next();
                if (jl + 1 < ri.nt) ok = issue(&map_k, ri, check_block(w1, ri));
                if (ok) ok = issue(&map_v, ri, check_block(w0, ri));
                w0 = w1;
                w1 = w2;
                w2 = w3;
            }
        }
        if (!ok && lane == 0) {
            for (uint32_t j = (slot_it > kNSlot ? slot_it - kNSlot : 0); j < slot_it; ++j)
                mbar_wait(&sh->slot_full[j % kNSlot], (j / kNSlot) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ======================= MMA issuer (one thread) =======================
        if (elect_one()) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kQRows, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kQRows, 1, 0);
            const uint32_t slot_addr = smem_u32(sSlot), q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            uint32_t slot_it = 0, q_it = 0, s_it = 0, p_it = 0;
            bool ok = true;
            auto do_pv = [&](bool first) -> bool {
                const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
                const uint32_t pb = p_it % kNP, pround = p_it / kNP;
                if (!mbar_wait(&sh->slot_full[st], round & 1, abort_flag)) return false;
                if (!mbar_wait(&sh->p_full[pb], pround & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t a0 = slot_addr + st * kSlotBytes;
                const uint32_t b0 = p_addr + pb * kPBytes;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int ks = 0; ks < kRowsTile / 16; ++ks) {
                        // V^T, MN-major: 64-d runs at LBO 1 KB (chunks of a block), 8-row groups at SBO 4 KB
                        const uint64_t ad = sdesc_sw128(a0 + (2 * ks) * kBlockBytes + half * 2048, 1024, kBlockBytes);
                        const uint64_t bd = sdesc_sw128(b0 + (ks >> 2) * kPChunk + (ks & 3) * 32, 16, 1024);
                        mma_bf16_ss(tmem + kOCol + half * 32, ad, bd, idesc_pv, (first && ks == 0) ? 0u : 1u);
                    }
                }
                mma_commit(&sh->slot_empty[st]);
                mma_commit(&sh->p_empty[pb]);
                ++slot_it;
                ++p_it;
                return true;
            };
            for (int64_t item = it_begin; ok && item < it_end; item += it_step) {
                const RowInfo ri = item_info(item);
                if (ri.nt == 0) continue;
                ok = mbar_wait(&sh->q_full, q_it & 1, abort_flag);
                ++q_it;
                const int nt = ri.nt;
                for (int jl = 0; ok && jl < nt; ++jl) {
                    const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
                    const uint32_t sb = s_it & 1, sround = s_it >> 1;
                    if (!(ok = mbar_wait(&sh->slot_full[st], round & 1, abort_flag))) break;
                    if (!(ok = mbar_wait(&sh->s_empty[sb], (sround & 1) ^ 1, abort_flag))) break;
                    tc_fence_after();
                    const uint32_t a0 = slot_addr + st * kSlotBytes;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t off = (ks & 3) * 32;
                        const uint64_t ad = sdesc_sw128(a0 + (ks >> 2) * 1024 + off, 16, kBlockBytes);
                        const uint64_t bd = sdesc_sw128(q_addr + (ks >> 2) * kQChunk + off, 16, 1024);
                        mma_bf16_ss(tmem + kSCol + sb * 32, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&sh->slot_empty[st]);
                    mma_commit(&sh->s_full[sb]);
                    ++slot_it;
                    ++s_it;
                    if (jl == nt - 1) mma_commit(&sh->q_empty);
                    if (jl >= 1) ok = do_pv(jl == 1);
                }
                if (ok) ok = do_pv(nt == 1);
                if (ok) mma_commit(&sh->o_full);
            }
        }
    } else {
        // ======================= softmax + epilogue (warps 2..5) =======================
        const int quad = warp & 3;
        const int R = quad * 32 + lane;               // TMEM lane: row of the tile
        const int blk_slot = R >> 3;                  // block within the tile
        const int tok_in_blk = (R >> 1) & 3;
        const int g = R & 1;                          // KV group of this row
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float c2 = scale * 1.4426950408889634f;
        const float rescale_raw = kRescaleLog2 / c2;
        const uint32_t p_addr = smem_u32(sP);
        const uint32_t p_row_off = (R >> 6) * kPChunk + (R & 7) * 2;
        const int p_unit = (R & 63) >> 3;
        uint32_t p_it = 0, s_it = 0, tile_it = 0, o_it = 0;
        bool ok = true;
        for (int64_t item = it_begin; ok && item < it_end; item += it_step) {
            const RowInfo ri = item_info(item);
            const int64_t slot = ri.slot;  // partial-state slot (schedules that merge)
            if (ri.nt == 0) {
                if (nsplit > 1 && bounds == nullptr) {  // empty split: neutral partial state
                    float *part = ws + slot * kHQ * kD;
                    for (int x = R; x < kHQ * kD; x += 128) part[x] = 0.f;
                    if (R < kHQ) ws[(size_t)n_slots * kHQ * kD + slot * kHQ + R] = -INFINITY;
                }
                continue;
            }
            const int nt = ri.nt;
            float m[kHQ];                             // running max per head (raw logits), identical in all threads
            float l[kGrp];                            // this row's share of the row sums, own group's heads
            float mc[kGrp];                           // own group: m * scale * log2(e)
#pragma unroll
            for (int h = 0; h < kGrp; ++h) l[h] = 0.f;
#pragma unroll
            for (int h = 0; h < kHQ; ++h) m[h] = 0.f;
            // raw ids two tiles ahead, checked at use (the producer flags bad ids)
            int32_t raw0 = load_block(sel, ri, kb, ri.p0 + blk_slot);
            int32_t raw1 = nt > 1 ? load_block(sel, ri, kb, ri.p0 + kBlkTile + blk_slot) : kNoBlock;
            for (int jl = 0; ok && jl < nt; ++jl) {
                const int32_t blk = check_block(raw0, ri);
                raw0 = raw1;
                raw1 = jl + 2 < nt ? load_block(sel, ri, kb, ri.p0 + (jl + 2) * kBlkTile + blk_slot) : kNoBlock;
                const bool valid = blk >= 0 && (int64_t)blk * r + tok_in_blk <= ri.t;
                const uint32_t sb = s_it & 1, sround = s_it >> 1;
                if (!(ok = mbar_wait(&sh->s_full[sb], sround & 1, abort_flag))) break;
                tc_fence_after();
                float s[kHQ];  // columns 0..23: the real heads (24..31 pad)
                tmem_ld16(tmem + lane_addr + kSCol + sb * 32, s);
                tmem_ld8(tmem + lane_addr + kSCol + sb * 32 + 16, s + 16);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&sh->s_empty[sb]);
                ++s_it;
                float v[kGrp];
#pragma unroll
                for (int h = 0; h < kGrp; ++h) v[h] = valid ? (g ? s[kGrp + h] : s[h]) : -INFINITY;
                // The running max only moves when some logit of the tile exceeds it by the
                // lazy-rescale margin (or on the item's first tile).  Every row tests its own
                // heads and one barrier ORs the answers; only then is the exact per-head tile
                // max reduced over the 128 rows.
                bool full = jl == 0;
                if (!full) {
                    bool ex = false;
#pragma unroll
                    for (int h = 0; h < kGrp; ++h) ex |= fmaf(v[h], c2, -mc[h]) > kRescaleLog2;
                    full = softmax_any(ex);
                }
                if (full) {
                    // exact per-head tile max: lanes of equal parity hold the same group
                    float tm[kGrp];
#pragma unroll
                    for (int h = 0; h < kGrp; ++h) {
                        float x = v[h];
                        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
                        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
                        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
                        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
                        tm[h] = x;
                    }
                    const int par = tile_it & 1;
                    if (lane < 2) {
#pragma unroll
                        for (int h = 0; h < kGrp; ++h) sh->red_max[par][quad][lane][h] = tm[h];
                    }
                    softmax_bar();
                    float tmax[kHQ];
#pragma unroll
                    for (int h = 0; h < kHQ; ++h) {
                        const int gg = h / kGrp, hh = h % kGrp;
                        tmax[h] = fmaxf(fmaxf(sh->red_max[par][0][gg][hh], sh->red_max[par][1][gg][hh]),
                                        fmaxf(sh->red_max[par][2][gg][hh], sh->red_max[par][3][gg][hh]));
                    }
                    ++tile_it;
                    if (jl == 0) {
#pragma unroll
                        for (int h = 0; h < kHQ; ++h) m[h] = tmax[h] == -INFINITY ? 0.f : tmax[h];
                    } else {
                        bool need = false;
#pragma unroll
                        for (int h = 0; h < kHQ; ++h) need |= tmax[h] > m[h] + rescale_raw;
                        if (need) {  // uniform: every thread computed the same maxima
                            float f[32];
#pragma unroll
                            for (int h = 0; h < 32; ++h) f[h] = 1.f;
#pragma unroll
                            for (int h = 0; h < kHQ; ++h) {
                                const float mn = fmaxf(m[h], tmax[h]);
                                f[h] = exp2f((m[h] - mn) * c2);
                                m[h] = mn;
                            }
#pragma unroll
                            for (int h = 0; h < kGrp; ++h) l[h] *= g ? f[kGrp + h] : f[h];
                            // O^T must be stable: wait for the previous PV (the completion of the
                            // last use of its P buffer), then scale it in TMEM
                            {
                                const uint32_t x = p_it - 1;
                                if (!(ok = mbar_wait(&sh->p_empty[x % kNP], (x / kNP) & 1, abort_flag))) break;
                            }
                            tc_fence_after();
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                float o[32];
                                const uint32_t ta = tmem + lane_addr + kOCol + half * 32;
                                tmem_ld32(ta, o);
                                tmem_wait_ld();
#pragma unroll
                                for (int h = 0; h < 32; ++h) o[h] *= f[h];
                                tmem_st32(ta, o);
                            }
                            tmem_wait_st();
                        }
                    }
#pragma unroll
                    for (int h = 0; h < kGrp; ++h) {
                        mc[h] = (g ? m[kGrp + h] : m[h]) * c2;
                    }
                }
                // P = exp(S - m) for the row's own-group heads; the rest of P^T stays zero
                const uint32_t pb = p_it % kNP, pround = p_it / kNP;
                if (!(ok = mbar_wait(&sh->p_empty[pb], (pround & 1) ^ 1, abort_flag))) break;
                const uint32_t pbase = p_addr + pb * kPBytes + p_row_off;
#pragma unroll
                for (int h = 0; h < kGrp; ++h) {
                    const float p = exp2f(fmaf(v[h], c2, -mc[h]));  // v = -inf (masked) gives 0
                    l[h] += p;
                    const int hq = g * kGrp + h;
                    const uint32_t addr = pbase + (hq >> 3) * 1024 + (hq & 7) * 128 + ((p_unit ^ (hq & 7)) << 4);
                    st_shared_b16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(p)));
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&sh->p_full[pb]);
                ++p_it;
            }
            if (!ok) break;
            // row sums: reduce the own-group heads over rows of equal parity, then over the 4 quads
#pragma unroll
            for (int h = 0; h < kGrp; ++h) {
                float x = l[h];
                x += __shfl_xor_sync(0xffffffffu, x, 16);
                x += __shfl_xor_sync(0xffffffffu, x, 8);
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                x += __shfl_xor_sync(0xffffffffu, x, 2);
                l[h] = x;
            }
            if (lane < 2) {
#pragma unroll
                for (int h = 0; h < kGrp; ++h) sh->red_sum[quad][lane][h] = l[h];
            }
            softmax_bar();
            float inv[kHQ];
            float mR = 0.f, LR = 1.f;  // thread R < 24 writes head R's log-sum-exp
#pragma unroll
            for (int h = 0; h < kHQ; ++h) {
                const int gg = h / kGrp, hh = h % kGrp;
                const float L = sh->red_sum[0][gg][hh] + sh->red_sum[1][gg][hh] + sh->red_sum[2][gg][hh] +
                                sh->red_sum[3][gg][hh];
                inv[h] = L > 0.f ? 1.f / L : 0.f;
                if (R == h) {
                    mR = m[h];
                    LR = L;
                }
            }
            const float my_lse = mR * scale + logf(LR);
            if (!(ok = mbar_wait(&sh->o_full, o_it & 1, abort_flag))) break;
            ++o_it;
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[32];
                tmem_ld32(tmem + lane_addr + kOCol + half * 32, o);
                tmem_wait_ld();
                const int d = half * 128 + R;
                if (!partials) {
                    __nv_bfloat16 *dst = out + ri.row * kHQ * kD + d;
#pragma unroll
                    for (int h = 0; h < kHQ; ++h) dst[h * kD] = __float2bfloat16_rn(o[h] * inv[h]);
                } else {
                    float *dst = ws + (slot * kHQ) * kD + d;
#pragma unroll
                    for (int h = 0; h < kHQ; ++h) __stcs(dst + h * kD, o[h] * inv[h]);
                }
            }
            if (R < kHQ) {
                if (!partials) {
                    if (lse_out != nullptr) lse_out[ri.row * kHQ + R] = my_lse;
                } else {
                    ws[(size_t)n_slots * kHQ * kD + slot * kHQ + R] = my_lse;
                }
            }
            tc_fence_before();
            softmax_bar();  // red_sum reuse by the next item
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}


// ---------------------------------------------------------------------------
// Decode kernel: the same attention for one query per sequence under the even
// schedule, with a pipeline made for keys that all come from DRAM.  Each CTA
// holds only three 64 KB slots, and per tile the V slot waited for the softmax
// of its tile and the next K waited behind that PV, so little of the ring was in
// flight.  Here an item's tiles go in chunks of up to kCT:
//   * all S of a chunk land in TMEM (two chunk buffers), the softmax reduces one
//     per-head max for the chunk and only then writes P tile by tile;
//   * the ring order is K of chunk 0, then for every tile u of chunk q: V(q, u),
//     K(q + 1, u) -- so a K slot frees as soon as its S MMA runs and a V slot as
//     soon as it lands (P is ready by then): the ring stays in flight.
constexpr int kCT = 7;                                  // tiles per chunk
constexpr uint32_t kDecSBuf = kCT * kQRows;             // TMEM columns of one chunk of S
constexpr uint32_t kDecOCol = 2 * kDecSBuf;             // O^T after two chunk buffers (448)
constexpr uint32_t kDecTmemCols = 512;
static_assert(kDecOCol + 64 <= kDecTmemCols, "two chunks of S and O^T fit in TMEM");

__global__ void __launch_bounds__(kAttThreads, 1)
sparse_decode_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const int32_t *__restrict__ sel,
                     const int32_t *__restrict__ cu_k, int64_t rows, int kb, int r, float scale,
                     float *__restrict__ ws, const int32_t *__restrict__ block_table, int page_size,
                     int max_pages, int64_t num_pages)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sSlot = smem;
    uint8_t *sQ = smem + kOffQ;
    uint8_t *sP = smem + kOffP;
    AttShared *sh = reinterpret_cast<AttShared *>(smem + kOffShared);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row_begin = 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNSlot; ++i) {
            mbar_init(&sh->slot_full[i], 1);
            mbar_init(&sh->slot_empty[i], 1);
        }
        mbar_init(&sh->q_full, 1);
        mbar_init(&sh->q_empty, 1);
        for (int i = 0; i < kNP; ++i) {
            mbar_init(&sh->p_full[i], 128);
            mbar_init(&sh->p_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->sc_full[i], 1);
            mbar_init(&sh->sc_empty[i], 128);
        }
        mbar_init(&sh->o_full, 1);
        sh->abort_flag = 0;
        fence_barrier_init();
    }
    // P^T entries of the other KV group and of the pad heads stay zero for good
    for (int i = threadIdx.x; i < kNP * kPBytes / 16; i += kAttThreads)
        reinterpret_cast<uint4 *>(sP)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, kDecTmemCols);
        tmem_relinquish();
    }
    if (warp == 2)
        even_setup(sh, cu_k, row_begin, rows, kb, r, lane,
                   reinterpret_cast<int64_t *>(ws + ((size_t)gridDim.x + rows) * kHQ * (kD + 1)));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    volatile int *abort_flag = &sh->abort_flag;
    const int64_t n_items = sh->ev_nseg;
    const int64_t n_slots = (int64_t)gridDim.x + rows;

    if (warp == 0) {
        // ======================= TMA producer (whole warp) =======================
        if (lane == 0) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_k);
            tma_prefetch_desc(&map_v);
        }
        uint32_t slot_it = 0, q_it = 0;
        bool ok = true;
        auto issue = [&](const CUtensorMap *map, const RowInfo &ri, int32_t blk) -> bool {
            const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
            bool good = true;
            if (lane == 0) {
                good = mbar_wait(&sh->slot_empty[st], (round & 1) ^ 1, abort_flag);
                if (good) mbar_arrive_expect_tx(&sh->slot_full[st], kSlotBytes);
            }
            good = __shfl_sync(0xffffffffu, good, 0);
            if (!good) return false;
            if (lane < kBlkTile) {
                // the block's first token row (token, group) in the cache; -8 reads zeros
                int32_t y = -8;
                if (blk >= 0) {
                    const int64_t tok = (int64_t)blk * r;  // position in the sequence
                    if (block_table == nullptr) {
                        y = (int32_t)((ri.tok_base + tok) * kHKV);
                    } else {
                        const int64_t j = tok / page_size;
                        const int32_t page = j < max_pages ? __ldg(block_table + ri.row * max_pages + j) : -1;
                        if (page >= 0 && page < num_pages)
                            y = (int32_t)(((int64_t)page * page_size + tok % page_size) * kHKV);
                        else
                            set_device_status(QSA_ERR_DEVICE_CHECK);
                    }
                }
                tma_load_3d(sSlot + st * kSlotBytes + lane * kBlockBytes, map, &sh->slot_full[st], 0, y, 0);
            }
            ++slot_it;
            return true;
        };
        for (int64_t item = 0; ok && item < n_items; ++item) {
            const RowInfo ri = row_info_even(item, sh, cu_k, row_begin, kb, r);
            if (ri.nt == 0) continue;
            const int nt = ri.nt, nch = (nt + kCT - 1) / kCT;
            int32_t cur[kCT], nxt[kCT];
#pragma unroll
            for (int u = 0; u < kCT; ++u)
                cur[u] = (lane < kBlkTile && u < nt) ? load_block(sel, ri, kb, ri.p0 + u * kBlkTile + lane) : kNoBlock;
            if (lane == 0) {
                ok = mbar_wait(&sh->q_empty, (q_it & 1) ^ 1, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(&sh->q_full, kQBytes);
                    for (int c = 0; c < 4; ++c)
                        tma_load_2d(sQ + c * kQChunk, &map_q, &sh->q_full, c * 64, (int32_t)(ri.row * kHQ));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ++q_it;
            const int len0 = nt < kCT ? nt : kCT;
#pragma unroll
            for (int u = 0; u < kCT; ++u)
                if (ok && u < len0) ok = issue(&map_k, ri, check_block(cur[u], ri));
            for (int q = 0; ok && q < nch; ++q) {
                const int len = nt - q * kCT < kCT ? nt - q * kCT : kCT;
                const int rest = nt - (q + 1) * kCT;
                const int lenn = rest <= 0 ? 0 : (rest < kCT ? rest : kCT);
#pragma unroll
                for (int u = 0; u < kCT; ++u)
                    nxt[u] = (lane < kBlkTile && u < lenn)
                                 ? load_block(sel, ri, kb, ri.p0 + ((q + 1) * kCT + u) * kBlkTile + lane)
                                 : kNoBlock;
#pragma unroll
                for (int u = 0; u < kCT; ++u) {
                    if (ok && u < len) ok = issue(&map_v, ri, check_block(cur[u], ri));
                    if (ok && u < lenn) ok = issue(&map_k, ri, check_block(nxt[u], ri));
                }
#pragma unroll
                for (int u = 0; u < kCT; ++u) cur[u] = nxt[u];
            }
        }
        if (!ok && lane == 0) {
            for (uint32_t j = (slot_it > kNSlot ? slot_it - kNSlot : 0); j < slot_it; ++j)
                mbar_wait(&sh->slot_full[j % kNSlot], (j / kNSlot) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ======================= MMA issuer (one thread) =======================
        if (elect_one()) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kQRows, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kQRows, 1, 0);
            const uint32_t slot_addr = smem_u32(sSlot), q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            uint32_t slot_it = 0, q_it = 0, p_it = 0, cc = 0;
            bool ok = true;
            auto do_s = [&](uint32_t buf, int u) -> bool {  // S of tile u of the chunk in buffer buf
                const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
                if (!mbar_wait(&sh->slot_full[st], round & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t a0 = slot_addr + st * kSlotBytes;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks & 3) * 32;
                    const uint64_t ad = sdesc_sw128(a0 + (ks >> 2) * 1024 + off, 16, kBlockBytes);
                    const uint64_t bd = sdesc_sw128(q_addr + (ks >> 2) * kQChunk + off, 16, 1024);
                    mma_bf16_ss(tmem + buf * kDecSBuf + u * kQRows, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(&sh->slot_empty[st]);
                ++slot_it;
                return true;
            };
            auto do_pv = [&](bool first) -> bool {
                const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
                const uint32_t pb = p_it % kNP, pround = p_it / kNP;
                if (!mbar_wait(&sh->slot_full[st], round & 1, abort_flag)) return false;
                if (!mbar_wait(&sh->p_full[pb], pround & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t a0 = slot_addr + st * kSlotBytes;
                const uint32_t b0 = p_addr + pb * kPBytes;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int ks = 0; ks < kRowsTile / 16; ++ks) {
                        const uint64_t ad = sdesc_sw128(a0 + (2 * ks) * kBlockBytes + half * 2048, 1024, kBlockBytes);
                        const uint64_t bd = sdesc_sw128(b0 + (ks >> 2) * kPChunk + (ks & 3) * 32, 16, 1024);
                        mma_bf16_ss(tmem + kDecOCol + half * 32, ad, bd, idesc_pv, (first && ks == 0) ? 0u : 1u);
                    }
                }
                mma_commit(&sh->slot_empty[st]);
                mma_commit(&sh->p_empty[pb]);
                ++slot_it;
                ++p_it;
                return true;
            };
            for (int64_t item = 0; ok && item < n_items; ++item) {
                const RowInfo ri = row_info_even(item, sh, cu_k, row_begin, kb, r);
                if (ri.nt == 0) continue;
                const int nt = ri.nt, nch = (nt + kCT - 1) / kCT;
                ok = mbar_wait(&sh->q_full, q_it & 1, abort_flag);
                ++q_it;
                // S of chunk 0 (its buffer must be free: chunk cc - 2 consumed)
                const int len0 = nt < kCT ? nt : kCT;
                if (ok) ok = mbar_wait(&sh->sc_empty[cc & 1], ((cc >> 1) & 1) ^ 1, abort_flag);
                for (int u = 0; ok && u < len0; ++u) ok = do_s(cc & 1, u);
                if (!ok) break;
                mma_commit(&sh->sc_full[cc & 1]);
                if (nch == 1) mma_commit(&sh->q_empty);
                for (int q = 0; ok && q < nch; ++q) {
                    const uint32_t cq = cc + q, cn = cq + 1;
                    const int len = nt - q * kCT < kCT ? nt - q * kCT : kCT;
                    const int rest = nt - (q + 1) * kCT;
                    const int lenn = rest <= 0 ? 0 : (rest < kCT ? rest : kCT);
                    if (lenn > 0) ok = mbar_wait(&sh->sc_empty[cn & 1], ((cn >> 1) & 1) ^ 1, abort_flag);
                    for (int u = 0; ok && u < len; ++u) {
                        ok = do_pv(q == 0 && u == 0);
                        if (ok && u < lenn) ok = do_s(cn & 1, u);
                    }
                    if (ok && lenn > 0) {
                        mma_commit(&sh->sc_full[cn & 1]);
                        if (q + 1 == nch - 1) mma_commit(&sh->q_empty);
                    }
                }
                if (ok) mma_commit(&sh->o_full);
                cc += nch;
            }
        }
    } else {
        // ======================= softmax + epilogue (warps 2..5) =======================
        const int quad = warp & 3;
        const int R = quad * 32 + lane;               // TMEM lane: row of the tile
        const int blk_slot = R >> 3;                  // block within the tile
        const int tok_in_blk = (R >> 1) & 3;
        const int g = R & 1;                          // KV group of this row
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float c2 = scale * 1.4426950408889634f;
        const float rescale_raw = kRescaleLog2 / c2;
        const uint32_t p_addr = smem_u32(sP);
        const uint32_t p_row_off = (R >> 6) * kPChunk + (R & 7) * 2;
        const int p_unit = (R & 63) >> 3;
        uint32_t p_it = 0, cc = 0, o_it = 0, red_it = 0;
        bool ok = true;
        for (int64_t item = 0; ok && item < n_items; ++item) {
            const RowInfo ri = row_info_even(item, sh, cu_k, row_begin, kb, r);
            const int64_t slot = ri.slot;
            if (ri.nt == 0) continue;
            const int nt = ri.nt, nch = (nt + kCT - 1) / kCT;
            float m[kHQ];     // running max per head (raw logits), identical in all threads
            float l[kGrp];    // this row's share of the row sums, own group's heads
            float mc[kGrp];   // own group: m * scale * log2(e)
#pragma unroll
            for (int h = 0; h < kGrp; ++h) l[h] = 0.f;
#pragma unroll
            for (int h = 0; h < kHQ; ++h) m[h] = 0.f;
            for (int q = 0; ok && q < nch; ++q, ++cc) {
                const uint32_t buf = cc & 1;
                const int len = nt - q * kCT < kCT ? nt - q * kCT : kCT;
                // which rows of the chunk's tiles count: a block past the range, an id out
                // of range (flagged by the producer) or a token after t does not
                uint32_t vmask = 0u;
#pragma unroll
                for (int u = 0; u < kCT; ++u) {
                    if (u < len) {
                        const int32_t blk = check_block(load_block(sel, ri, kb, ri.p0 + (q * kCT + u) * kBlkTile + blk_slot), ri);
                        if (blk >= 0 && (int64_t)blk * r + tok_in_blk <= ri.t) vmask |= 1u << u;
                    }
                }
                if (!(ok = mbar_wait(&sh->sc_full[buf], (cc >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                // phase A: the chunk's per-head max over its 128 x len rows
                float tm[kGrp];
#pragma unroll
                for (int h = 0; h < kGrp; ++h) tm[h] = -INFINITY;
#pragma unroll
                for (int u = 0; u < kCT; ++u) {
                    if (u < len) {
                        float s[kHQ];
                        tmem_ld16(tmem + lane_addr + buf * kDecSBuf + u * kQRows, s);
                        tmem_ld8(tmem + lane_addr + buf * kDecSBuf + u * kQRows + 16, s + 16);
                        tmem_wait_ld();
                        if (vmask & (1u << u)) {
#pragma unroll
                            for (int h = 0; h < kGrp; ++h) tm[h] = fmaxf(tm[h], g ? s[kGrp + h] : s[h]);
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < kGrp; ++h) {  // lanes of equal parity hold the same group
                    float x = tm[h];
                    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
                    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
                    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
                    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
                    tm[h] = x;
                }
                const int par = red_it & 1;
                if (lane < 2) {
#pragma unroll
                    for (int h = 0; h < kGrp; ++h) sh->red_max[par][quad][lane][h] = tm[h];
                }
                softmax_bar();
                ++red_it;
                float tmax[kHQ];
#pragma unroll
                for (int h = 0; h < kHQ; ++h) {
                    const int gg = h / kGrp, hh = h % kGrp;
                    tmax[h] = fmaxf(fmaxf(sh->red_max[par][0][gg][hh], sh->red_max[par][1][gg][hh]),
                                    fmaxf(sh->red_max[par][2][gg][hh], sh->red_max[par][3][gg][hh]));
                }
                if (q == 0) {
#pragma unroll
                    for (int h = 0; h < kHQ; ++h) m[h] = tmax[h] == -INFINITY ? 0.f : tmax[h];
                } else {
                    bool need = false;
#pragma unroll
                    for (int h = 0; h < kHQ; ++h) need |= tmax[h] > m[h] + rescale_raw;
                    if (need) {  // uniform: every thread computed the same maxima
                        float f[32];
#pragma unroll
                        for (int h = 0; h < 32; ++h) f[h] = 1.f;
#pragma unroll
                        for (int h = 0; h < kHQ; ++h) {
                            const float mn = fmaxf(m[h], tmax[h]);
                            f[h] = exp2f((m[h] - mn) * c2);
                            m[h] = mn;
                        }
#pragma unroll
                        for (int h = 0; h < kGrp; ++h) l[h] *= g ? f[kGrp + h] : f[h];
                        {  // every PV so far has completed once the last P buffer used is released
                            const uint32_t x = p_it - 1;
                            if (!(ok = mbar_wait(&sh->p_empty[x % kNP], (x / kNP) & 1, abort_flag))) break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            float o[32];
                            const uint32_t ta = tmem + lane_addr + kDecOCol + half * 32;
                            tmem_ld32(ta, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int h = 0; h < 32; ++h) o[h] *= f[h];
                            tmem_st32(ta, o);
                        }
                        tmem_wait_st();
                    }
                }
#pragma unroll
                for (int h = 0; h < kGrp; ++h) mc[h] = (g ? m[kGrp + h] : m[h]) * c2;
                // phase B: P = exp(S - m) tile by tile, for the PVs as their V lands
#pragma unroll
                for (int u = 0; u < kCT; ++u) {
                    if (!ok || u >= len) continue;
                    const uint32_t pb = p_it % kNP, pround = p_it / kNP;
                    if (!(ok = mbar_wait(&sh->p_empty[pb], (pround & 1) ^ 1, abort_flag))) continue;
                    float s[kHQ];
                    tmem_ld16(tmem + lane_addr + buf * kDecSBuf + u * kQRows, s);
                    tmem_ld8(tmem + lane_addr + buf * kDecSBuf + u * kQRows + 16, s + 16);
                    tmem_wait_ld();
                    const bool valid = (vmask >> u) & 1u;
                    const uint32_t pbase = p_addr + pb * kPBytes + p_row_off;
#pragma unroll
                    for (int h = 0; h < kGrp; ++h) {
                        const float x = g ? s[kGrp + h] : s[h];
                        const float p = valid ? exp2f(fmaf(x, c2, -mc[h])) : 0.f;
                        l[h] += p;
                        const int hq = g * kGrp + h;
                        const uint32_t addr = pbase + (hq >> 3) * 1024 + (hq & 7) * 128 + ((p_unit ^ (hq & 7)) << 4);
                        st_shared_b16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(p)));
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(&sh->p_full[pb]);
                    ++p_it;
                }
                if (!ok) break;
                tc_fence_before();
                mbar_arrive(&sh->sc_empty[buf]);  // this chunk's S is read: the buffer may be refilled
            }
            if (!ok) break;
            // row sums: reduce the own-group heads over rows of equal parity, then over the 4 quads
#pragma unroll
            for (int h = 0; h < kGrp; ++h) {
                float x = l[h];
                x += __shfl_xor_sync(0xffffffffu, x, 16);
                x += __shfl_xor_sync(0xffffffffu, x, 8);
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                x += __shfl_xor_sync(0xffffffffu, x, 2);
                l[h] = x;
            }
            if (lane < 2) {
#pragma unroll
                for (int h = 0; h < kGrp; ++h) sh->red_sum[quad][lane][h] = l[h];
            }
            softmax_bar();
            float inv[kHQ];
            float mR = 0.f, LR = 1.f;
#pragma unroll
            for (int h = 0; h < kHQ; ++h) {
                const int gg = h / kGrp, hh = h % kGrp;
                const float L = sh->red_sum[0][gg][hh] + sh->red_sum[1][gg][hh] + sh->red_sum[2][gg][hh] +
                                sh->red_sum[3][gg][hh];
                inv[h] = L > 0.f ? 1.f / L : 0.f;
                if (R == h) {
                    mR = m[h];
                    LR = L;
                }
            }
            if (!(ok = mbar_wait(&sh->o_full, o_it & 1, abort_flag))) break;
            ++o_it;
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[32];
                tmem_ld32(tmem + lane_addr + kDecOCol + half * 32, o);
                tmem_wait_ld();
                float *dst = ws + (slot * kHQ) * kD + half * 128 + R;
#pragma unroll
                for (int h = 0; h < kHQ; ++h) __stcs(dst + h * kD, o[h] * inv[h]);
            }
            if (R < kHQ) ws[(size_t)n_slots * kHQ * kD + slot * kHQ + R] = mR * scale + logf(LR);
            tc_fence_before();
            softmax_bar();  // red_sum reuse by the next item
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kDecTmemCols);
    }
}

// merge split-K partials: lse = logsumexp_s lse_s, o = sum_s exp(lse_s - lse) o_s;
// with bounds, splits (key chunks) whose selection range is empty hold no state
__global__ void __launch_bounds__(256)
combine_kernel(const float *__restrict__ ws, int64_t n_items, int nsplit, const int32_t *__restrict__ bounds,
               __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out)
{
    const int64_t row = blockIdx.x;
    const int h = blockIdx.y;
    const int d = threadIdx.x;
    const float *lp = ws + (size_t)n_items * kHQ * kD + row * nsplit * kHQ + h;
    const int32_t *bd = bounds ? bounds + row * (nsplit + 1) : nullptr;
    float mx = -INFINITY;
    for (int s = 0; s < nsplit; ++s)
        if (bd == nullptr || bd[s + 1] > bd[s]) mx = fmaxf(mx, lp[s * kHQ]);
    float tot = 0.f, acc = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        if (bd != nullptr && bd[s + 1] <= bd[s]) continue;
        const float l = lp[s * kHQ];
        const float wgt = (l == -INFINITY) ? 0.f : __expf(l - mx);
        tot += wgt;
        acc += wgt * __ldcs(ws + ((row * nsplit + s) * kHQ + h) * kD + d);
    }
    out[(row * kHQ + h) * kD + d] = __float2bfloat16_rn(tot > 0.f ? acc / tot : 0.f);
    if (lse_out != nullptr && d == 0) lse_out[row * kHQ + h] = mx + logf(tot);
}

// merge the pieces of each row under the even schedule: the piece at the row's first
// tile (slot grid + row) and one per share that starts inside the row and holds tiles
// (slot = share).  The rows' first tiles come from the attention kernel (CTA 0).
__global__ void __launch_bounds__(256)
even_combine_kernel(const float *__restrict__ ws, int grid, int64_t row_begin, int64_t rows,
                    __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out)
{
    const int64_t rl = blockIdx.x;
    const int h = blockIdx.y;
    const int d = threadIdx.x;
    const int64_t n_slots = (int64_t)grid + rows;
    const float *lbase = ws + (size_t)n_slots * kHQ * kD;
    const int64_t *tile_prefix = reinterpret_cast<const int64_t *>(ws + (size_t)n_slots * kHQ * (kD + 1));
    const int64_t total = tile_prefix[rows], rs = tile_prefix[rl], re = tile_prefix[rl + 1];
    __nv_bfloat16 *dst = out + ((row_begin + rl) * kHQ + h) * kD + d;
    if (re <= rs) {  // an empty sequence: nothing attended
        *dst = __float2bfloat16_rn(0.f);
        if (lse_out != nullptr && d == 0) lse_out[(row_begin + rl) * kHQ + h] = -INFINITY;
        return;
    }
    auto share_start = [&](int64_t c) { return c * total / grid; };
    auto piece = [&](int64_t c) { return share_start(c) > rs && share_start(c + 1) > share_start(c); };
    const int64_t c0 = rs * grid / total;
    float mx = lbase[((int64_t)grid + rl) * kHQ + h];
    for (int64_t c = c0; c < grid && share_start(c) < re; ++c)
        if (piece(c)) mx = fmaxf(mx, lbase[c * kHQ + h]);
    float tot = 0.f, acc = 0.f;
    auto add = [&](int64_t slot) {
        const float l = lbase[slot * kHQ + h];
        const float wgt = (l == -INFINITY) ? 0.f : __expf(l - mx);
        tot += wgt;
        acc += wgt * __ldcs(ws + (slot * kHQ + h) * kD + d);
    };
    add((int64_t)grid + rl);
    for (int64_t c = c0; c < grid && share_start(c) < re; ++c)
        if (piece(c)) add(c);
    *dst = __float2bfloat16_rn(tot > 0.f ? acc / tot : 0.f);
    if (lse_out != nullptr && d == 0) lse_out[(row_begin + rl) * kHQ + h] = mx + logf(tot);
}

// key-chunk boundaries of each row's (ascending) selection: bounds[rl][c] = number of
// selected blocks below c * chunk_blocks, c = 0 .. nchunks (one warp per row)
__global__ void __launch_bounds__(256)
chunk_bounds_kernel(const int32_t *__restrict__ sel, const int32_t *__restrict__ cu_q,
                    const int32_t *__restrict__ cu_k, int batch, int64_t row_begin, int64_t rows, int kb, int r,
                    int chunk_blocks, int nchunks, int32_t *__restrict__ bounds)
{
    const int lane = threadIdx.x & 31;
    const int64_t rl = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (rl >= rows) return;
    const int64_t row = row_begin + rl;
    const int s = find_seq(cu_q, batch, row);
    const int64_t Lq = (int64_t)cu_q[s + 1] - cu_q[s];
    const int64_t Lk = (int64_t)cu_k[s + 1] - cu_k[s];
    const int64_t t = (Lk - Lq) + (row - cu_q[s]);
    int32_t *bd = bounds + rl * (nchunks + 1);
    if (t < 0) {
        for (int c = lane; c <= nchunks; c += 32) bd[c] = 0;
        return;
    }
    const int64_t bt = t / r;
    const int nsel = (int)(bt + 1 < kb ? bt + 1 : kb);
    const int32_t *srow = sel + row * kb;
    auto chunk_of = [&](int j) -> int {
        const int32_t b = __ldg(srow + j);
        if (b < 0) return 0;
        const int c = b / chunk_blocks;
        return c < nchunks ? c : nchunks - 1;
    };
    // position j starts its chunk when the previous entry lies in a lower chunk:
    // bounds[c] = j for every c in (chunk(j - 1), chunk(j)]
    for (int j = lane; j < nsel; j += 32) {
        const int cj = chunk_of(j);
        const int cprev = j > 0 ? chunk_of(j - 1) : -1;
        for (int c = cprev + 1; c <= cj; ++c) bd[c] = j;
        if (j == nsel - 1)
            for (int c = cj + 1; c <= nchunks; ++c) bd[c] = nsel;
    }
}

}  // namespace

int min_nsplit(int kb)
{
    (void)kb;
    return 1;  // the online softmax handles any budget in one pass
}

int dense_decode_nsplit(int64_t max_len_k, int r)
{
    const int64_t blocks = (max_len_k + r - 1) / r;
    const int64_t tiles = (blocks + kBlkTile - 1) / kBlkTile;
    const int64_t ns = (tiles + 31) / 32;  // about 2048 tokens per split, as a QSA query
    return (int)(ns > 0 ? ns : 1);
}

int even_grid()
{
    const int g = num_sms();
    return g < kMaxEvenCtas ? g : kMaxEvenCtas;
}

size_t even_workspace_bytes(int64_t rows, int grid)
{
    // partial states (o, lse) of rows + grid slots, then the rows' first tiles
    return (size_t)(rows + grid) * kHQ * (kD + 1) * sizeof(float) + (size_t)(rows + 1) * sizeof(int64_t);
}

size_t split_workspace_bytes(int64_t rows, int nsplit)
{
    return nsplit > 1 ? (size_t)rows * nsplit * kHQ * (kD + 1) * sizeof(float) : 0;
}

size_t chunked_workspace_bytes(int64_t rows, int nchunks)
{
    const size_t b = ((size_t)rows * (nchunks + 1) * sizeof(int32_t) + 255) & ~(size_t)255;
    return b + split_workspace_bytes(rows, nchunks);
}

cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0) return cudaSuccess;
    const bool chunked = a.nchunks > 1;
    const int nsplit = chunked ? a.nchunks : a.nsplit;
    if (nsplit > 1 && a.ws == nullptr) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    // q as [rows_total * 24, 256], 32-row boxes (24 heads + 8 rows of padding)
    if (!make_tmap_2d(&mq, a.q, kD, (uint64_t)a.total_q * kHQ, kD * 2, 64, kQRows)) return cudaErrorInvalidValue;
    // k, v as (64 d, token-row, 4 d-chunks) with strides (512 B, 128 B): one box = one micro-block
    if (!make_tmap_3d(&mk, a.k, 64, (uint64_t)a.total_k * kHKV, 4, kD * 2, 128, 64, 8, 4)) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mv, a.v, 64, (uint64_t)a.total_k * kHKV, 4, kD * 2, 128, 64, 8, 4)) return cudaErrorInvalidValue;
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
        attr = true;
    }
    float *ws = a.ws;
    int32_t *bounds = nullptr;
    if (chunked) {
        bounds = reinterpret_cast<int32_t *>(a.ws);
        const size_t bb = ((size_t)rows * (a.nchunks + 1) * sizeof(int32_t) + 255) & ~(size_t)255;
        ws = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.ws) + bb);
        chunk_bounds_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
            a.sel, a.cu_q, a.cu_k, a.batch, a.row_begin, rows, a.kb, a.r, a.chunk_blocks, a.nchunks, bounds);
    }
    if (a.even) {  // decode, even schedule: shares of the batch's tiles, then the merge
        if (a.cu_q != nullptr || a.ws == nullptr || chunked || nsplit != 1) return cudaErrorInvalidValue;
        const int grid = even_grid();
        static bool dattr = false;
        if (!dattr) {
            cudaFuncSetAttribute(sparse_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
            dattr = true;
        }
        if (a.row_begin != 0) return cudaErrorInvalidValue;
        if (a.block_table != nullptr && (a.page_size <= 0 || a.page_size % a.r != 0 || a.max_pages <= 0))
            return cudaErrorInvalidValue;
        sparse_decode_kernel<<<(unsigned)grid, kAttThreads, kAttSmem, stream>>>(
            mq, mk, mv, a.sel, a.cu_k, rows, a.kb, a.r, a.scale, ws, a.block_table, a.page_size, a.max_pages,
            a.block_table != nullptr ? a.total_k / a.page_size : 0);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        even_combine_kernel<<<dim3((unsigned)rows, kHQ), kD, 0, stream>>>(ws, grid, a.row_begin, rows, a.o,
                                                                          a.lse);
        return cudaGetLastError();
    }
    const int64_t n_items = rows * nsplit;
    int64_t grid = num_sms();
    if (grid > n_items) grid = n_items;
    sparse_attn_kernel<<<(unsigned)grid, kAttThreads, kAttSmem, stream>>>(
        mq, mk, mv, a.sel, a.cu_q, a.cu_k, a.batch, a.row_begin, rows, nsplit, a.kb, a.r, a.scale, a.o, a.lse,
        ws, bounds);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || nsplit == 1) return e;
    dim3 cg((unsigned)rows, kHQ);
    combine_kernel<<<cg, kD, 0, stream>>>(ws, n_items, nsplit, bounds, a.o + a.row_begin * kHQ * kD,
                                          a.lse ? a.lse + a.row_begin * kHQ : nullptr);
    return cudaGetLastError();
}

}  // namespace qsa
