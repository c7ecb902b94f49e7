// attn_common.cuh -- shared pieces of the QSA attention kernels (prefill in
// attn.cu, decode in attn_decode.cu): tile constants, the shared-memory layout,
// work items of the three prefill schedules and of the even decode schedule,
// block-id loads and checks, and small PTX helpers.  Only those two files
// include it.
#pragma once
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

}  // namespace

}  // namespace qsa
