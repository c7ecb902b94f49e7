// attn.cu -- QSA sparse GQA core attention: prefill (and split-K dense decode).
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
//                  epilogue (thread = d); the split-K dense decode and the
//                  key-chunked schedule write fp32 partial states that
//                  combine_kernel merges.
// Without a selection array the kernel attends to every block j <= t: that is
// the dense flash-decoding baseline (one query per sequence, split-K).
#include "attn_common.cuh"

namespace qsa {

namespace {

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
    {
        const cudaError_t e = set_smem_attr_once(reinterpret_cast<const void *>(sparse_attn_kernel), kAttSmem);
        if (e != cudaSuccess) return e;
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
    if (a.even) return launch_sparse_decode(a, stream);  // decode: attn_decode.cu
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
