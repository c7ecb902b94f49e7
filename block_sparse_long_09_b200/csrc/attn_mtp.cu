// attn_mtp.cu -- QSA sparse GQA attention for a decode step with multi-token
// prediction: next_n <= 4 new queries per sequence (t = L - next_n .. L - 1) share
// ONE selection of micro-blocks.
//
// "On the Design of Qwen3.8 Next Architecture" (reading notes): "结果 2" measures
// decode with next_n = 4 (three MTP prediction steps), and section 5, step 5,
// says the MTP steps reuse the QSA top-k indices; the attention itself is the
// sparse core attention of section 6 (query t sees the tokens j <= t of the
// selected blocks).  One gathered K/V tile then serves all next_n queries, so
// the step reads each sequence's 2048 selected tokens once for next_n tokens.
//
// Layout ("standard" orientation): the next_n x 24 query heads are the MMA's M
// side (96 of 128 rows; the rest are zero and ignored), the tile's 128 K/V rows
// (16 micro-blocks x 4 tokens x 2 KV heads, one 4 KB TMA box per block) its N
// side, so a thread owns one (query, head) row and its softmax needs no
// cross-thread reduction:
//   S = Q K^T   M128 N128 K256 (both K-major), S double-buffered in TMEM
//   O += P V    M128 N256 K128 (P K-major from shared memory, V MN-major)
// A row's key columns of the other KV group, blocks past the selection and tokens
// after the row's own position are masked.  Online softmax with a lazy rescale
// of the row's O in TMEM (only when its max grows by more than 2^8).
// Warp roles: 0 TMA producer (Q per item, then K and V tiles, one slot each),
// 1 TMEM owner and MMA issuer (S(j) runs one tile ahead of PV(j - 1)), 2..5 the
// softmax and epilogue.  A sequence's tiles are split over several CTAs (work
// items); their partial (o, lse) states are merged by mtp_combine_kernel.
// TMEM: S 2 x 128 columns + O 256.  Shared memory: Q 64 KB, P 32 KB, K and V
// 64 KB each.
#include "attn_common.cuh"

namespace qsa {

namespace {

constexpr int kMaxNQ = 4;
constexpr int kMRows = kMaxNQ * kHQ;              // 96 (query, head) rows
constexpr int kQChunkM = 128 * 128;               // 16 KB: 64 d-columns x 128 rows
constexpr int kQBytesM = 4 * kQChunkM;            // 64 KB
constexpr int kMtpBlk = 8;                        // micro-blocks per tile
constexpr int kMtpKeys = kMtpBlk * 8;             // 64 K/V rows per tile: 8 blocks x 4 tokens x 2 groups
constexpr int kMtpSlot = kMtpBlk * kBlockBytes;   // 32 KB: one tile of K (or V)
constexpr int kPBufM = 128 * 128;                 // 16 KB: P of one tile, 64 key columns x 128 rows
constexpr int kMtpThreads = 192;
constexpr uint32_t kMtpSCol = 0, kMtpOCol = 256, kMtpTmemCols = 512;

struct MtpShared {
    uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
    uint64_t q_full, q_empty;
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2], p_empty[2];
    uint64_t o_full, o_empty;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr int kOffKM = kQBytesM;
constexpr int kOffVM = kOffKM + 2 * kMtpSlot;
constexpr int kOffPM = kOffVM + 2 * kMtpSlot;
constexpr int kOffShM = kOffPM + 2 * kPBufM;
constexpr int kMtpSmem = kOffShM + (int)sizeof(MtpShared) + 1024;
static_assert(kMtpSmem <= 232448, "shared memory of one CTA");

struct MtpItem {
    int64_t s;       // sequence
    int sp;          // split
    int64_t L, tok_base;
    int64_t b_last;  // own block of the last query
    int nsel;        // valid entries of the shared selection
    int p0, nt;      // first selection position and tiles of this item
};

// the shared selection of sequence s holds min(b_first, k - nf) + nf blocks
__device__ __forceinline__ MtpItem mtp_item(int64_t item, int nsplit, const int32_t *cu_k, int kb, int r, int next_n)
{
    MtpItem it;
    it.s = item / nsplit;
    it.sp = (int)(item % nsplit);
    it.tok_base = __ldg(cu_k + it.s);
    it.L = (int64_t)__ldg(cu_k + it.s + 1) - it.tok_base;
    it.nt = 0;
    it.p0 = 0;
    it.nsel = 0;
    it.b_last = 0;
    if (it.L <= 0) return it;
    const int64_t t_first = it.L - next_n > 0 ? it.L - next_n : 0;
    const int64_t b_first = t_first / r;
    it.b_last = (it.L - 1) / r;
    const int64_t nf = it.b_last - b_first + 1;
    const int64_t room = kb - nf > 0 ? kb - nf : 0;
    it.nsel = (int)((b_first < room ? b_first : room) + nf);
    if (it.nsel > kb) it.nsel = kb;
    const int tiles = (it.nsel + kMtpBlk - 1) / kMtpBlk;
    const int tps = (tiles + nsplit - 1) / nsplit;
    const int a = it.sp * tps, b = (it.sp + 1) * tps < tiles ? (it.sp + 1) * tps : tiles;
    it.p0 = a * kMtpBlk;
    it.nt = b > a ? b - a : 0;
    return it;
}

__global__ void __launch_bounds__(kMtpThreads, 1)
sparse_mtp_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const int32_t *__restrict__ sel,
                  const int32_t *__restrict__ cu_k, int batch, int next_n, int nsplit, int kb, int r,
                  float scale, __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out,
                  float *__restrict__ ws, const int32_t *__restrict__ block_table, int page_size, int max_pages,
                  int64_t num_pages)
{
    pdl_enter();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = smem + kOffKM;
    uint8_t *sV = smem + kOffVM;
    uint8_t *sP = smem + kOffPM;
    MtpShared *sh = reinterpret_cast<MtpShared *>(smem + kOffShM);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh->k_full[i], 1);
            mbar_init(&sh->k_empty[i], 1);
            mbar_init(&sh->v_full[i], 1);
            mbar_init(&sh->v_empty[i], 1);
            mbar_init(&sh->s_full[i], 1);
            mbar_init(&sh->s_empty[i], 128);
            mbar_init(&sh->p_full[i], 128);
            mbar_init(&sh->p_empty[i], 1);
        }
        mbar_init(&sh->q_full, 1);
        mbar_init(&sh->q_empty, 1);
        mbar_init(&sh->o_full, 1);
        mbar_init(&sh->o_empty, 128);
        sh->abort_flag = 0;
        fence_barrier_init();
    }
    // the Q rows the TMA never writes (96..127) start at zero; P is written whole per tile
    for (int i = threadIdx.x; i < kQBytesM / 16; i += kMtpThreads)
        if ((i * 16) % kQChunkM >= kMRows * 128) reinterpret_cast<uint4 *>(sQ)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, kMtpTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    volatile int *abort_flag = &sh->abort_flag;
    const int64_t n_items = (int64_t)batch * nsplit;
    const bool partials = nsplit > 1;

    if (warp == 0) {
        // ======================= TMA producer (whole warp) =======================
        if (lane == 0) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_k);
            tma_prefetch_desc(&map_v);
        }
        uint32_t ku = 0, vu = 0, qu = 0;
        bool ok = true;
        // one ring use: lane 0 waits for the slot and arms its barrier, lanes 0..7 load a block each
        auto issue = [&](const CUtensorMap *map, uint8_t *ring, uint64_t *full, uint64_t *empty, uint32_t use,
                         const MtpItem &it, int32_t raw) -> bool {
            const uint32_t st = use & 1;
            bool good = true;
            if (lane == 0) {
                good = mbar_wait(&empty[st], ((use >> 1) & 1) ^ 1, abort_flag);
                if (good) mbar_arrive_expect_tx(&full[st], kMtpSlot);
            }
            good = __shfl_sync(0xffffffffu, good, 0);
            if (!good) return false;
            if (lane < kMtpBlk) {
                int32_t y = -8;  // reads zeros
                if (raw != kNoBlock) {
                    if (raw < 0 || raw > it.b_last) {
                        set_device_status(QSA_ERR_DEVICE_CHECK);
                    } else {
                        const int64_t tok = (int64_t)raw * r;
                        if (block_table == nullptr) {
                            y = (int32_t)((it.tok_base + tok) * kHKV);
                        } else {
                            const int64_t j = tok / page_size;
                            const int32_t page = j < max_pages ? __ldg(block_table + it.s * max_pages + j) : -1;
                            if (page >= 0 && page < num_pages)
                                y = (int32_t)(((int64_t)page * page_size + tok % page_size) * kHKV);
                            else
                                set_device_status(QSA_ERR_DEVICE_CHECK);
                        }
                    }
                }
                tma_load_3d(ring + st * kMtpSlot + lane * kBlockBytes, map, &full[st], 0, y, 0);
            }
            return true;
        };
        for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const MtpItem it = mtp_item(item, nsplit, cu_k, kb, r, next_n);
            if (it.nt == 0) continue;
            if (lane == 0) {
                ok = mbar_wait(&sh->q_empty, (qu & 1) ^ 1, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(&sh->q_full, kMRows * 128 * 4);
                    for (int c = 0; c < 4; ++c)
                        tma_load_2d(sQ + c * kQChunkM, &map_q, &sh->q_full, c * 64,
                                    (int32_t)(it.s * next_n * kHQ));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ++qu;
            auto tile_id = [&](int j) {  // this lane's block of tile j (lanes 0..7)
                const int pos = it.p0 + j * kMtpBlk + lane;
                return (lane < kMtpBlk && j < it.nt && pos < it.nsel) ? __ldg(sel + it.s * kb + pos) : kNoBlock;
            };
            int32_t raw = tile_id(0);
            for (int j = 0; ok && j < it.nt; ++j) {
                const int32_t raw_next = tile_id(j + 1);  // in flight while tile j is issued
                ok = issue(&map_k, sK, sh->k_full, sh->k_empty, ku++, it, raw);
                if (ok) ok = issue(&map_v, sV, sh->v_full, sh->v_empty, vu++, it, raw);
                raw = raw_next;
            }
        }
        if (!ok && lane == 0) {  // let every copy in flight land before the CTA exits
            for (uint32_t u = (ku > 2 ? ku - 2 : 0); u < ku; ++u) mbar_wait(&sh->k_full[u & 1], (u >> 1) & 1, nullptr);
            for (uint32_t u = (vu > 2 ? vu - 2 : 0); u < vu; ++u) mbar_wait(&sh->v_full[u & 1], (u >> 1) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ======================= MMA issuer (one thread) =======================
        if (elect_one()) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kMtpKeys, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kD, 0, 1);
            const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV),
                           p_addr = smem_u32(sP);
            uint32_t ku = 0, vu = 0, qu = 0, su = 0, pu = 0, ou = 0;
            bool ok = true;
            auto do_s = [&]() -> bool {  // S = Q K^T of the next K tile into S buffer su & 1
                const uint32_t sb = su & 1, kb_ = ku & 1;
                if (!mbar_wait(&sh->k_full[kb_], (ku >> 1) & 1, abort_flag)) return false;
                if (!mbar_wait(&sh->s_empty[sb], ((su >> 1) & 1) ^ 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k0 = k_addr + kb_ * kMtpSlot;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks & 3) * 32;
                    const uint64_t ad = sdesc_sw128(q_addr + (ks >> 2) * kQChunkM + off, 16, 1024);
                    const uint64_t bd = sdesc_sw128(k0 + (ks >> 2) * 1024 + off, 16, kBlockBytes);
                    mma_bf16_ss(tmem + kMtpSCol + sb * kMtpKeys, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(&sh->k_empty[kb_]);
                mma_commit(&sh->s_full[sb]);
                ++ku;
                ++su;
                return true;
            };
            auto do_pv = [&](bool first) -> bool {  // O += P V of the next V tile
                const uint32_t vb = vu & 1, pb = pu & 1;
                if (!mbar_wait(&sh->v_full[vb], (vu >> 1) & 1, abort_flag)) return false;
                if (!mbar_wait(&sh->p_full[pb], (pu >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t v0 = v_addr + vb * kMtpSlot, p0 = p_addr + pb * kPBufM;
#pragma unroll
                for (int ks = 0; ks < kMtpKeys / 16; ++ks) {
                    const uint64_t ad = sdesc_sw128(p0 + ks * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(v0 + (2 * ks) * kBlockBytes, 1024, kBlockBytes);
                    mma_bf16_ss(tmem + kMtpOCol, ad, bd, idesc_pv, (first && ks == 0) ? 0u : 1u);
                }
                mma_commit(&sh->v_empty[vb]);
                mma_commit(&sh->p_empty[pb]);
                ++vu;
                ++pu;
                return true;
            };
            for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const MtpItem it = mtp_item(item, nsplit, cu_k, kb, r, next_n);
                if (it.nt == 0) continue;
                ok = mbar_wait(&sh->q_full, qu & 1, abort_flag);
                ++qu;
                if (ok) ok = do_s();
                if (ok && it.nt == 1) mma_commit(&sh->q_empty);
                // the item's first PV overwrites O: the previous item's epilogue must have read it
                if (ok) ok = mbar_wait(&sh->o_empty, (ou & 1) ^ 1, abort_flag);
                for (int j = 0; ok && j < it.nt; ++j) {
                    if (j + 1 < it.nt) {
                        ok = do_s();
                        if (ok && j + 2 == it.nt) mma_commit(&sh->q_empty);
                    }
                    if (ok) ok = do_pv(j == 0);
                }
                if (ok) mma_commit(&sh->o_full);
                ++ou;
            }
        }
    } else {
        // ======================= softmax + epilogue (warps 2..5) =======================
        const int quad = warp & 3;
        const int R = quad * 32 + lane;   // TMEM lane = (query, head) row
        const bool live = R < next_n * kHQ;
        const int qi = R / kHQ, h = R % kHQ, g = h / kGrp;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float c2 = scale * 1.4426950408889634f;
        const float margin = kRescaleLog2 / c2;  // lazy rescale threshold, raw logit units
        const uint32_t p_row = smem_u32(sP) + R * 128;
        uint32_t su = 0, pu = 0, ou = 0;
        bool ok = true;
        for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const MtpItem it = mtp_item(item, nsplit, cu_k, kb, r, next_n);
            const int64_t slot = item;
            if (it.nt == 0) {  // an empty split: a neutral partial state (an empty sequence: zeros)
                if (partials && live) {
                    float *part = ws + (slot * kMRows + R) * kD;
                    for (int d = 0; d < kD; ++d) part[d] = 0.f;
                    ws[(size_t)n_items * kMRows * kD + slot * kMRows + R] = -INFINITY;
                } else if (live) {
                    __nv_bfloat16 *dst = out + ((it.s * next_n + qi) * kHQ + h) * kD;
                    for (int d = 0; d < kD; ++d) dst[d] = __float2bfloat16_rn(0.f);
                    if (lse_out != nullptr) lse_out[(it.s * next_n + qi) * kHQ + h] = -INFINITY;
                }
                continue;
            }
            const int64_t t = it.L - next_n + qi;  // this row's position
            float m = -INFINITY, l = 0.f;
            for (int j = 0; ok && j < it.nt; ++j) {
                const uint32_t sb = su & 1;
                if (!(ok = mbar_wait(&sh->s_full[sb], (su >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                float s[kMtpKeys];
                __syncwarp();
#pragma unroll
                for (int c = 0; c < kMtpKeys / 32; ++c)
                    tmem_ld32(tmem + lane_addr + kMtpSCol + sb * kMtpKeys + c * 32, s + c * 32);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&sh->s_empty[sb]);
                ++su;
                // which key columns this row sees: its KV group, a selected block, token <= t
                const int pbase = it.p0 + j * kMtpBlk;
                float mt = -INFINITY;
#pragma unroll
                for (int bs = 0; bs < kMtpBlk; ++bs) {
                    const int pos = pbase + bs;
                    const int32_t blk = pos < it.nsel ? __ldg(sel + it.s * kb + pos) : -1;
                    const bool bok = live && blk >= 0 && blk <= it.b_last;
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {  // column bs * 8 + c8 = (token c8 / 2, KV group c8 % 2)
                        const int c = bs * 8 + c8;
                        const bool v = bok && (c8 & 1) == g && (int64_t)blk * r + (c8 >> 1) <= t;
                        s[c] = v ? s[c] : -INFINITY;
                        mt = fmaxf(mt, s[c]);
                    }
                }
                // the running maxima move when some row of the warp grows by more than the margin
                // (and on the first tile); O is then rescaled by the whole warp once every earlier
                // PV has landed (rows whose maximum stayed put scale by 1)
                if (__any_sync(0xffffffffu, mt > m + margin || j == 0)) {
                    const float mn = fmaxf(m, mt);
                    if (j > 0) {
                        {  // PV(j - 1) used P buffer (pu - 1) & 1: its completion covers every PV before it
                            const uint32_t x = pu - 1;
                            if (!(ok = mbar_wait(&sh->p_empty[x & 1], (x >> 1) & 1, abort_flag))) break;
                        }
                        tc_fence_after();
                        const float f = mn == -INFINITY ? 1.f : exp2f((m - mn) * c2);
                        l *= f;
#pragma unroll 1
                        for (int c = 0; c < kD / 32; ++c) {
                            float o[32];
                            const uint32_t ta = tmem + lane_addr + kMtpOCol + c * 32;
                            tmem_ld32(ta, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int x = 0; x < 32; ++x) o[x] *= f;
                            tmem_st32(ta, o);
                        }
                        tmem_wait_st();
                    }
                    m = mn;
                }
                // P(j) goes to buffer pu & 1, free once PV(j - 2) has completed
                {
                    const uint32_t pb = pu & 1;
                    if (!(ok = mbar_wait(&sh->p_empty[pb], ((pu >> 1) & 1) ^ 1, abort_flag))) break;
                    tc_fence_after();
                    const float mc = (m == -INFINITY ? 0.f : m) * c2;
                    // P row: own-group columns exp(S - m), the rest 0; 128-byte swizzled K-major layout
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = u * 8 + e * 2;
                            const float p0 = exp2f(fmaf(s[c], c2, -mc));      // -inf gives 0
                            const float p1 = exp2f(fmaf(s[c + 1], c2, -mc));
                            l += p0 + p1;
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                            pk[e] = *reinterpret_cast<const uint32_t *>(&b2);
                        }
                        const uint32_t addr = p_row + pb * kPBufM + ((u ^ (R & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[0]),
                                     "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(&sh->p_full[pb]);
                    ++pu;
                }
            }
            if (!ok) break;
            // epilogue: O / l of this row
            if (!(ok = mbar_wait(&sh->o_full, ou & 1, abort_flag))) break;
            ++ou;
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float my_lse = (m == -INFINITY || l <= 0.f) ? -INFINITY : m * scale + logf(l);
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                float o[32];
                __syncwarp();  // the TMEM load is a warp-wide instruction
                tmem_ld32(tmem + lane_addr + kMtpOCol + c * 32, o);
                tmem_wait_ld();
                if (!live) continue;
                if (!partials) {
                    __nv_bfloat16 *dst = out + ((it.s * next_n + qi) * kHQ + h) * kD + c * 32;
#pragma unroll
                    for (int x = 0; x < 32; x += 8) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(o[x + 2 * e] * inv, o[x + 2 * e + 1] * inv);
                            pk[e] = *reinterpret_cast<const uint32_t *>(&b2);
                        }
                        *reinterpret_cast<uint4 *>(dst + x) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                } else {
                    float *dst = ws + (slot * kMRows + R) * kD + c * 32;
#pragma unroll
                    for (int x = 0; x < 32; x += 4)
                        __stcs(reinterpret_cast<float4 *>(dst + x),
                               make_float4(o[x] * inv, o[x + 1] * inv, o[x + 2] * inv, o[x + 3] * inv));
                }
            }
            tc_fence_before();
            mbar_arrive(&sh->o_empty);
            if (live) {
                if (!partials) {
                    if (lse_out != nullptr) lse_out[(it.s * next_n + qi) * kHQ + h] = my_lse;
                } else {
                    ws[(size_t)n_items * kMRows * kD + slot * kMRows + R] = my_lse;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kMtpTmemCols);
    }
}

// merge the splits of each (sequence, query row): lse = logsumexp of the parts,
// o = sum exp(lse_part - lse) o_part / sum exp(lse_part - lse).  A warp per row: lane sp
// holds split sp's weight (nsplit <= 32), each lane 8 of the 256 dims.
constexpr int kCombRows = 8;  // rows (warps) per CTA

__global__ void __launch_bounds__(kCombRows * 32)
mtp_combine_kernel(const float *__restrict__ ws, int64_t n_items, int nsplit, int next_n,
                   __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out)
{
    pdl_enter();
    const int64_t s = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int R = blockIdx.y * kCombRows + (threadIdx.x >> 5);  // (query, head) row
    if (R >= next_n * kHQ) return;  // warp-uniform
    const float *lp = ws + (size_t)n_items * kMRows * kD + (s * nsplit) * kMRows + R;
    const float *pp = ws + ((s * nsplit) * kMRows + R) * kD + lane;
    const float l = lane < nsplit ? lp[lane * kMRows] : -INFINITY;
    float mx = l;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float wgt = (l == -INFINITY) ? 0.f : __expf(l - mx);
    float tot = 0.f, acc[kD / 32];
#pragma unroll
    for (int i = 0; i < kD / 32; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int sp = 0; sp < nsplit; ++sp) {  // the splits in order
        const float w = __shfl_sync(0xffffffffu, wgt, sp);
        tot += w;
        float o[kD / 32];
#pragma unroll
        for (int i = 0; i < kD / 32; ++i) o[i] = __ldcs(pp + (size_t)sp * kMRows * kD + i * 32);
#pragma unroll
        for (int i = 0; i < kD / 32; ++i) acc[i] += w * o[i];
    }
    const int qi = R / kHQ, h = R % kHQ;
    __nv_bfloat16 *dst = out + ((s * next_n + qi) * kHQ + h) * kD + lane;
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
#pragma unroll
    for (int i = 0; i < kD / 32; ++i) dst[i * 32] = __float2bfloat16_rn(tot > 0.f ? acc[i] * inv : 0.f);
    if (lse_out != nullptr && lane == 0) lse_out[(s * next_n + qi) * kHQ + h] = tot > 0.f ? mx + logf(tot) : -INFINITY;
}

}  // namespace

int mtp_nsplit(int batch, int kb)
{
    // splits per sequence: the fewest that minimise the busiest CTA's work in tile units,
    // ceil(batch * ns / G) items of tiles / ns tiles each, plus the partial states that
    // splits write and the merge reads back (96 x 257 fp32 twice: about 3 tiles of K/V
    // bytes each), spread over the G CTAs
    const int tiles = (kb + kMtpBlk - 1) / kMtpBlk;
    const int64_t G = num_sms();
    if (batch <= 0) return 1;
    int best = 1;
    double best_cost = -1.0;
    for (int ns = 1; ns <= tiles && ns <= 32; ++ns) {  // the merge keeps a split's weight per lane
        const int64_t items_per_cta = ((int64_t)batch * ns + G - 1) / G;
        const double cost = (double)(items_per_cta * ((tiles + ns - 1) / ns)) +
                            (ns > 1 ? 3.0 * (double)batch * ns / (double)G : 0.0);
        if (best_cost < 0.0 || cost < best_cost) {
            best = ns;
            best_cost = cost;
        }
    }
    return best;
}

size_t mtp_workspace_bytes(int batch, int kb)
{
    const int ns = mtp_nsplit(batch, kb);
    return ns > 1 ? (size_t)batch * ns * kMRows * (kD + 1) * sizeof(float) : 0;
}

cudaError_t launch_sparse_mtp(const AttnArgs &a, int next_n, cudaStream_t stream)
{
    const int64_t batch = a.batch;
    if (batch <= 0) return cudaSuccess;
    if (next_n < 1 || next_n > kMaxNQ) return cudaErrorInvalidValue;
    const int nsplit = mtp_nsplit((int)batch, a.kb);
    if (nsplit > 1 && a.ws == nullptr) return cudaErrorInvalidValue;
    if (a.block_table != nullptr && (a.page_size <= 0 || a.page_size % a.r != 0 || a.max_pages <= 0))
        return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    // q as [batch * next_n * 24, 256]: a sequence's next_n x 24 rows are one box (rows past them
    // belong to the next sequence or lie out of range and are never read back)
    if (!make_tmap_2d(&mq, a.q, kD, (uint64_t)batch * next_n * kHQ, kD * 2, 64, kMRows)) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mk, a.k, 64, (uint64_t)a.total_k * kHKV, 4, kD * 2, 128, 64, 8, 4)) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mv, a.v, 64, (uint64_t)a.total_k * kHKV, 4, kD * 2, 128, 64, 8, 4)) return cudaErrorInvalidValue;
    {
        const cudaError_t e = set_smem_attr_once(reinterpret_cast<const void *>(sparse_mtp_kernel), kMtpSmem);
        if (e != cudaSuccess) return e;
    }
    const int64_t n_items = batch * nsplit;
    int64_t grid = num_sms();
    if (grid > n_items) grid = n_items;
    cudaError_t e = launch_pdl(sparse_mtp_kernel, dim3((unsigned)grid), dim3(kMtpThreads), kMtpSmem, stream, mq, mk, mv,
                               a.sel, a.cu_k, (int)batch, next_n, nsplit, a.kb, a.r, a.scale, a.o, a.lse, a.ws,
                               a.block_table, a.page_size, a.max_pages,
                               a.block_table != nullptr ? a.total_k / a.page_size : (int64_t)0);
    if (e != cudaSuccess || nsplit == 1) return e;
    return launch_pdl(mtp_combine_kernel, dim3((unsigned)batch, (unsigned)((next_n * kHQ + kCombRows - 1) / kCombRows)),
                      dim3(kCombRows * 32), 0, stream, (const float *)a.ws, n_items, nsplit, next_n, a.o, a.lse);
}

}  // namespace qsa
