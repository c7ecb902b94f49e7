// attn_decode.cu -- QSA sparse GQA attention for decode: one new query per
// sequence, the selected tokens of the whole batch spread evenly over the CTAs.
//
// "On the Design of Qwen3.8 Next Architecture" (reading notes), section 6 and
// "结果 2": the same sparse core attention as the prefill, for the token each
// sequence is decoding.  The batch's 64-token tiles are cut into equal shares,
// one per CTA; a sequence cut by a share boundary is attended in pieces whose
// softmax states even_combine_kernel merges.
//
// The pipeline is made for keys that all come from DRAM.  A CTA has three
// 64 KB slots; a per-tile pipeline keeps each V slot until the softmax of its
// tile is done and the next K behind that PV, so little of the ring is in
// flight.  Here an item's tiles go in chunks of up to kCT:
//   * all S of a chunk land in TMEM (two chunk buffers), the softmax reduces one
//     per-head max for the chunk and only then writes P tile by tile;
//   * the ring order is K of chunk 0, then for every tile u of chunk q: V(q, u),
//     K(q + 1, u) -- so a K slot frees as soon as its S MMA runs and a V slot as
//     soon as it lands (P is ready by then): the ring stays in flight.
#include "attn_common.cuh"

namespace qsa {

namespace {

constexpr int kCT = 3;                                  // tiles per chunk (1 .. 7 fit TMEM; 2 to 4 measured
                                                        // ~7% faster than 7 at batch 64, 128K-256K context)
constexpr uint32_t kDecSBuf = kCT * kQRows;             // TMEM columns of one chunk of S
constexpr uint32_t kDecOCol = 2 * kDecSBuf;             // O^T after two chunk buffers
constexpr uint32_t kDecTmemCols = 512;
static_assert(kDecOCol + 64 <= kDecTmemCols, "two chunks of S and O^T fit in TMEM");

// The producer's TMA issue of one ring slot: lane 0 waits for the slot and arms its
// barrier, lanes 0..15 each load one block (its first token row in the packed cache,
// or through the block table; -8 reads zeros).  Called by the whole warp.
static __device__ __noinline__ bool dec_issue(const CUtensorMap *map, AttShared *sh, uint8_t *sSlot,
                                              uint32_t *slot_it, volatile int *abort_flag, int lane,
                                              int64_t tok_base, int64_t row, int32_t blk, int r,
                                              const int32_t *block_table, int page_size, int max_pages,
                                              int64_t num_pages)
{
    const uint32_t st = *slot_it % kNSlot, round = *slot_it / kNSlot;
    bool good = true;
    if (lane == 0) {
        good = mbar_wait(&sh->slot_empty[st], (round & 1) ^ 1, abort_flag);
        if (good) mbar_arrive_expect_tx(&sh->slot_full[st], kSlotBytes);
    }
    good = __shfl_sync(0xffffffffu, good, 0);
    if (!good) return false;
    if (lane < kBlkTile) {
        int32_t y = -8;
        if (blk >= 0) {
            const int64_t tok = (int64_t)blk * r;  // position in the sequence
            if (block_table == nullptr) {
                y = (int32_t)((tok_base + tok) * kHKV);
            } else {
                const int64_t j = tok / page_size;
                const int32_t page = j < max_pages ? __ldg(block_table + row * max_pages + j) : -1;
                if (page >= 0 && page < num_pages)
                    y = (int32_t)(((int64_t)page * page_size + tok % page_size) * kHKV);
                else
                    set_device_status(QSA_ERR_DEVICE_CHECK);
            }
        }
        tma_load_3d(sSlot + st * kSlotBytes + lane * kBlockBytes, map, &sh->slot_full[st], 0, y, 0);
    }
    ++*slot_it;
    return true;
}

// A selection entry as a block to attend: -1 when there is none, when it lies outside
// 0 .. b_t (flagged), or, for a context-parallel shard (blk_lo != nullptr), when it lies
// outside the shard's block window [blk_lo[row], blk_hi[row]) (not flagged: another
// shard holds it).
__device__ __forceinline__ int32_t dec_block(int32_t raw, const RowInfo &ri, const int32_t *blk_lo,
                                             const int32_t *blk_hi)
{
    int32_t b = check_block(raw, ri);
    if (b >= 0 && blk_lo != nullptr && (b < __ldg(blk_lo + ri.row) || b >= __ldg(blk_hi + ri.row))) b = -1;
    return b;
}

__global__ void __launch_bounds__(kAttThreads, 1)
sparse_decode_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const int32_t *__restrict__ sel,
                     const int32_t *__restrict__ cu_k, int64_t rows, int kb, int r, float scale,
                     float *__restrict__ ws, const int32_t *__restrict__ block_table, int page_size,
                     int max_pages, int64_t num_pages, const int64_t *__restrict__ tok_local,
                     const int32_t *__restrict__ blk_lo, const int32_t *__restrict__ blk_hi)
{
    pdl_enter();
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
        // one call site per ring slot use, 21 per chunk pair: a real call keeps the
        // producer's code small (the kernel's warps share the instruction cache)
        auto issue = [&](const CUtensorMap *map, const RowInfo &ri, int32_t blk) -> bool {
            // a shard's cache holds the window's tokens from tok_local[row] on
            const int64_t tok_base =
                tok_local != nullptr ? __ldg(tok_local + ri.row) - (int64_t)__ldg(blk_lo + ri.row) * r : ri.tok_base;
            return dec_issue(map, sh, sSlot, &slot_it, abort_flag, lane, tok_base, ri.row, blk, r, block_table,
                             page_size, max_pages, num_pages);
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
            // the block ids of chunk q + 1 are loaded while chunk q's copies are issued, so an
            // id load never stalls the issue of the copy that needs it
            auto load_chunk = [&](int q, int32_t (&ids)[kCT]) {
                const int rest = nt - q * kCT;
                const int len = rest <= 0 ? 0 : (rest < kCT ? rest : kCT);
#pragma unroll
                for (int u = 0; u < kCT; ++u)
                    ids[u] = (lane < kBlkTile && u < len) ? load_block(sel, ri, kb, ri.p0 + (q * kCT + u) * kBlkTile + lane)
                                                           : kNoBlock;
            };
            load_chunk(1, nxt);
            const int len0 = nt < kCT ? nt : kCT;
#pragma unroll
            for (int u = 0; u < kCT; ++u)
                if (ok && u < len0) ok = issue(&map_k, ri, dec_block(cur[u], ri, blk_lo, blk_hi));
            for (int q = 0; ok && q < nch; ++q) {
                const int len = nt - q * kCT < kCT ? nt - q * kCT : kCT;
                const int rest = nt - (q + 1) * kCT;
                const int lenn = rest <= 0 ? 0 : (rest < kCT ? rest : kCT);
                int32_t nxt2[kCT];
                load_chunk(q + 2, nxt2);
#pragma unroll
                for (int u = 0; u < kCT; ++u) {
                    if (ok && u < len) ok = issue(&map_v, ri, dec_block(cur[u], ri, blk_lo, blk_hi));
                    if (ok && u < lenn) ok = issue(&map_k, ri, dec_block(nxt[u], ri, blk_lo, blk_hi));
                }
#pragma unroll
                for (int u = 0; u < kCT; ++u) {
                    cur[u] = nxt[u];
                    nxt[u] = nxt2[u];
                }
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
                        const int32_t blk = dec_block(load_block(sel, ri, kb, ri.p0 + (q * kCT + u) * kBlkTile + blk_slot),
                                                      ri, blk_lo, blk_hi);
                        if (blk >= 0 && (int64_t)blk * r + tok_in_blk <= ri.t) vmask |= 1u << u;
                    }
                }
                if (!(ok = mbar_wait(&sh->sc_full[buf], (cc >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                // phase A: the chunk's per-head max over its 128 x len rows
                float tm[kGrp];
#pragma unroll
                for (int h = 0; h < kGrp; ++h) tm[h] = -INFINITY;
#pragma unroll 1
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
#pragma unroll 1
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

// merge the pieces of each row under the even schedule: the piece at the row's first
// tile (slot grid + row) and one per share that starts inside the row and holds tiles
// (slot = share).  The rows' first tiles come from the attention kernel (CTA 0).
// A warp per (row, head): its lanes find the row's pieces (32 shares at a time),
// reduce their log-sum-exps, then sum the partial outputs in piece order, 8 dims per lane.
constexpr int kMergeWarps = 8;  // heads per CTA (24 = 3 x 8)
static_assert(kHQ % kMergeWarps == 0, "whole heads per CTA");

__global__ void __launch_bounds__(kMergeWarps * 32)
even_combine_kernel(const float *__restrict__ ws, int grid, int64_t row_begin, int64_t rows,
                    __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out)
{
    pdl_enter();
    const int64_t rl = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y * kMergeWarps + (threadIdx.x >> 5);
    const int64_t n_slots = (int64_t)grid + rows;
    const float *lbase = ws + (size_t)n_slots * kHQ * kD;
    const int64_t *tile_prefix = reinterpret_cast<const int64_t *>(ws + (size_t)n_slots * kHQ * (kD + 1));
    const int64_t total = tile_prefix[rows], rs = tile_prefix[rl], re = tile_prefix[rl + 1];
    __nv_bfloat16 *dst = out + ((row_begin + rl) * kHQ + h) * kD + lane;
    if (re <= rs) {  // an empty sequence: nothing attended
#pragma unroll
        for (int i = 0; i < kD / 32; ++i) dst[i * 32] = __float2bfloat16_rn(0.f);
        if (lse_out != nullptr && lane == 0) lse_out[(row_begin + rl) * kHQ + h] = -INFINITY;
        return;
    }
    // the row's pieces: its first-tile slot (grid + rl), then every share c >= c0 that
    // starts inside the row and is not empty (share starts grow with c)
    auto share_start = [&](int64_t c) { return c * total / grid; };
    const int64_t c0 = rs * grid / total;
    auto is_piece = [&](int64_t c) {
        if (c >= grid) return false;
        const int64_t sc = share_start(c);
        return sc < re && sc > rs && share_start(c + 1) > sc;
    };
    const float l_first = lbase[((int64_t)grid + rl) * kHQ + h];
    float mx = l_first;
    for (int64_t cb = c0; cb < grid && share_start(cb) < re; cb += 32) {
        const int64_t c = cb + lane;
        if (is_piece(c)) mx = fmaxf(mx, lbase[c * kHQ + h]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float tot = 0.f, acc[kD / 32];
#pragma unroll
    for (int i = 0; i < kD / 32; ++i) acc[i] = 0.f;
    auto add = [&](int64_t slot, float l) {
        const float wgt = (l == -INFINITY) ? 0.f : __expf(l - mx);
        tot += wgt;
        const float *p = ws + (slot * kHQ + h) * kD + lane;
        float o[kD / 32];
#pragma unroll
        for (int i = 0; i < kD / 32; ++i) o[i] = __ldcs(p + i * 32);
#pragma unroll
        for (int i = 0; i < kD / 32; ++i) acc[i] += wgt * o[i];
    };
    add((int64_t)grid + rl, l_first);
    for (int64_t cb = c0; cb < grid && share_start(cb) < re; cb += 32) {
        const int64_t c = cb + lane;
        const bool mine = is_piece(c);
        const float lc = mine ? lbase[c * kHQ + h] : -INFINITY;
        uint32_t m = __ballot_sync(0xffffffffu, mine);
        // in share order, the partial outputs of up to four pieces loaded before they are
        // added (a small batch cuts a row into tens of pieces): the sums keep their order
        while (m != 0u) {
            constexpr int kAhead = 4;
            int src[kAhead];
            int cnt = 0;
#pragma unroll
            for (int j = 0; j < kAhead; ++j) {
                src[j] = m != 0u ? __ffs(m) - 1 : 0;
                if (m != 0u) {
                    m &= m - 1u;
                    ++cnt;
                }
            }
            float o[kAhead][kD / 32];
#pragma unroll
            for (int j = 0; j < kAhead; ++j) {
                if (j < cnt) {
                    const float *p = ws + ((cb + src[j]) * kHQ + h) * kD + lane;
#pragma unroll
                    for (int i = 0; i < kD / 32; ++i) o[j][i] = __ldcs(p + i * 32);
                }
            }
#pragma unroll
            for (int j = 0; j < kAhead; ++j) {
                const float l = __shfl_sync(0xffffffffu, lc, src[j]);
                if (j < cnt) {
                    const float wgt = (l == -INFINITY) ? 0.f : __expf(l - mx);
                    tot += wgt;
#pragma unroll
                    for (int i = 0; i < kD / 32; ++i) acc[i] += wgt * o[j][i];
                }
            }
        }
    }
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
#pragma unroll
    for (int i = 0; i < kD / 32; ++i) dst[i * 32] = __float2bfloat16_rn(tot > 0.f ? acc[i] * inv : 0.f);
    if (lse_out != nullptr && lane == 0) lse_out[(row_begin + rl) * kHQ + h] = mx + logf(tot);
}

// Context-parallel merge: the shards' normalised outputs o_p and log-sum-exps lse_p of
// the same (row, head) give o = sum_p exp(lse_p - lse) o_p, lse = log sum_p exp(lse_p).
// A warp per (row, head), 8 dims per lane, shards in order.
__global__ void __launch_bounds__(kMergeWarps * 32)
merge_states_kernel(const __nv_bfloat16 *__restrict__ o_parts, const float *__restrict__ lse_parts, int parts,
                    int64_t rows, __nv_bfloat16 *__restrict__ o, float *__restrict__ lse)
{
    const int64_t rl = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y * kMergeWarps + (threadIdx.x >> 5);
    const int64_t stride_o = rows * kHQ * kD, stride_l = rows * kHQ;
    float mx = -INFINITY;
    for (int p = lane; p < parts; p += 32) mx = fmaxf(mx, lse_parts[p * stride_l + rl * kHQ + h]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float tot = 0.f, acc[kD / 32];
#pragma unroll
    for (int i = 0; i < kD / 32; ++i) acc[i] = 0.f;
    for (int p = 0; p < parts; ++p) {
        const float l = lse_parts[p * stride_l + rl * kHQ + h];
        const float wgt = (l == -INFINITY) ? 0.f : __expf(l - mx);
        tot += wgt;
        const __nv_bfloat16 *src = o_parts + p * stride_o + (rl * kHQ + h) * kD + lane;
#pragma unroll
        for (int i = 0; i < kD / 32; ++i) acc[i] += wgt * __bfloat162float(src[i * 32]);
    }
    __nv_bfloat16 *dst = o + (rl * kHQ + h) * kD + lane;
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
#pragma unroll
    for (int i = 0; i < kD / 32; ++i) dst[i * 32] = __float2bfloat16_rn(acc[i] * inv);
    if (lse != nullptr && lane == 0) lse[rl * kHQ + h] = tot > 0.f ? mx + logf(tot) : -INFINITY;
}

}  // namespace

cudaError_t launch_sparse_decode(const AttnArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0) return cudaSuccess;
    if (a.cu_q != nullptr || a.ws == nullptr || a.nchunks > 1 || a.nsplit != 1 || a.row_begin != 0)
        return cudaErrorInvalidValue;
    if (a.block_table != nullptr && (a.page_size <= 0 || a.page_size % a.r != 0 || a.max_pages <= 0))
        return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    // q as [rows_total * 24, 256], 32-row boxes (24 heads + 8 rows of padding)
    if (!make_tmap_2d(&mq, a.q, kD, (uint64_t)a.total_q * kHQ, kD * 2, 64, kQRows)) return cudaErrorInvalidValue;
    // k, v as (64 d, token-row, 4 d-chunks) with strides (512 B, 128 B): one box = one micro-block
    if (!make_tmap_3d(&mk, a.k, 64, (uint64_t)a.total_k * kHKV, 4, kD * 2, 128, 64, 8, 4)) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mv, a.v, 64, (uint64_t)a.total_k * kHKV, 4, kD * 2, 128, 64, 8, 4)) return cudaErrorInvalidValue;
    {
        const cudaError_t e = set_smem_attr_once(reinterpret_cast<const void *>(sparse_decode_kernel), kAttSmem);
        if (e != cudaSuccess) return e;
    }
    const int grid = even_grid();
    cudaError_t e = launch_pdl(sparse_decode_kernel, dim3((unsigned)grid), dim3(kAttThreads), kAttSmem, stream, mq, mk,
                               mv, a.sel, a.cu_k, rows, a.kb, a.r, a.scale, a.ws, a.block_table, a.page_size,
                               a.max_pages, a.block_table != nullptr ? a.total_k / a.page_size : (int64_t)0,
                               a.tok_local, a.blk_lo, a.blk_hi);
    if (e != cudaSuccess) return e;
    return launch_pdl(even_combine_kernel, dim3((unsigned)rows, kHQ / kMergeWarps), dim3(kMergeWarps * 32), 0, stream,
                      (const float *)a.ws, grid, a.row_begin, rows, a.o, a.lse);
}

cudaError_t launch_merge_states(const __nv_bfloat16 *o_parts, const float *lse_parts, int parts, int64_t rows,
                                __nv_bfloat16 *o, float *lse, cudaStream_t stream)
{
    if (rows <= 0) return cudaSuccess;
    if (parts <= 0 || rows > 0x7FFFFFFF) return cudaErrorInvalidValue;
    merge_states_kernel<<<dim3((unsigned)rows, kHQ / kMergeWarps), kMergeWarps * 32, 0, stream>>>(
        o_parts, lse_parts, parts, rows, o, lse);
    return cudaGetLastError();
}

}  // namespace qsa
