// attn.cu -- QSA sparse GQA core attention (prefill and split-K decode).
//
// "On the Design of Qwen3.8 Next Architecture" (reading notes), section 6: the
// selected micro-blocks are expanded to their token indices and handed to the
// sparse core attention, O(nK) for a fixed budget K = 2048 tokens.  Heads per
// the "Model Summary" table: 24 query heads, 2 KV heads (12 query heads per
// group), head dim 256.  Query t sees the tokens of its selected blocks with
// j <= t (causal inside its own block).
//
// Design (B200): a persistent CTA per SM walks work items = (query row, split).
// For one item and one KV group g the 12 heads of g share every gathered key,
// so the contraction is laid out "swap-AB": keys are the M = 128 side of the
// tcgen05 MMA and the 12 heads (padded to N = 16) the N side, which keeps the
// tensor-core waste at 16/12 instead of 128/12.
//   warp 0      TMA producer: per 128-token tile and group, 32 micro-blocks x 4
//               d-chunks are gathered as 4-row boxes straight into the 128-byte
//               swizzled operand layout (3-slot ring of 64 KB); padding slots
//               load an out-of-range box, i.e. zeros.
//   warp 1      TMEM allocation + single-thread MMA issue:
//               S^T[key, head]  = K_tile[128 x 256] . Q_g^T          (K-major A and B)
//               O^T[d, head]   += V_tile^T[256 x 128] . P^T[128 x 16] (MN-major A)
//   warps 2..5  softmax: S^T of all <= 16 tiles of the group stays in TMEM
//               (16 columns each), so the exact per-head max is taken first and
//               P = exp(S - max) needs no rescaling; P^T goes to shared memory in
//               the swizzled K-major layout for the PV MMA; the epilogue reads O^T
//               back from TMEM, divides by the row sums and writes bf16 (or, for
//               split-K decode, fp32 partials + log-sum-exp for the combine kernel).
// The kernel is bound by the gather (4 MiB of K/V per query), not by the MMAs.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kHQ = 24, kHKV = 2, kD = 256, kGrp = kHQ / kHKV;
constexpr int kTileTok = 128;
constexpr int kBlkPerTile = 32;             // r = 4
constexpr int kMaxTiles = 16;               // budget 512 blocks = 2048 tokens
constexpr int kSlotBytes = kTileTok * kD * 2;   // 64 KB: one K or V tile of one group
constexpr int kChunk = kTileTok * 128;      // 16 KB: 64 d-columns of a tile
constexpr int kNSlot = 3;
constexpr int kQGroupBytes = 16 * kD * 2;   // 8 KB: 16 rows (12 heads + 4 pad) x 256
constexpr int kQBytes = 2 * kQGroupBytes;
constexpr int kPBytes = 16 * kTileTok * 2;  // 4 KB: P^T, 16 heads x 128 keys
constexpr int kNP = 2;
constexpr int kAttThreads = 192;
constexpr uint32_t kSCol = 0, kOCol = 256, kTmemCols = 512;

struct AttShared {
    uint64_t slot_full[kNSlot], slot_empty[kNSlot];
    uint64_t q_full, q_empty;
    uint64_t s_full, o_full;
    uint64_t p_full[kNP], p_empty[kNP];
    uint32_t tmem_base;
    int abort_flag;
    float red_max[4][16];
    float red_sum[4][16];
};

constexpr int kOffQ = kNSlot * kSlotBytes;
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kOffShared = kOffP + kNP * kPBytes;
constexpr int kAttSmem = kOffShared + (int)sizeof(AttShared) + 1024;

struct RowInfo {
    int64_t row;    // packed query row
    int s;
    int64_t t, bt, tok_base;
    int nsel, tile0, tile1;
    bool ok;
};

__device__ __forceinline__ RowInfo row_info(int64_t item, int nsplit, int64_t row_begin,
                                            const int32_t *cu_q, const int32_t *cu_k, int batch,
                                            int kb, int r)
{
    RowInfo ri;
    ri.row = row_begin + item / nsplit;
    const int sp = (int)(item % nsplit);
    if (cu_q != nullptr) {
        ri.s = find_seq(cu_q, batch, ri.row);
        const int64_t Lq = (int64_t)cu_q[ri.s + 1] - cu_q[ri.s];
        const int64_t Lk = (int64_t)cu_k[ri.s + 1] - cu_k[ri.s];
        ri.t = (Lk - Lq) + (ri.row - cu_q[ri.s]);
    } else {
        ri.s = (int)ri.row;
        ri.t = (int64_t)cu_k[ri.s + 1] - cu_k[ri.s] - 1;
    }
    ri.ok = ri.t >= 0;
    ri.bt = ri.ok ? ri.t / r : 0;
    ri.tok_base = cu_k[ri.s];
    const int64_t nsel = ri.bt + 1 < kb ? ri.bt + 1 : kb;
    ri.nsel = (int)nsel;
    const int ntiles = (int)((nsel + kBlkPerTile - 1) / kBlkPerTile);
    const int max_tiles = (kb + kBlkPerTile - 1) / kBlkPerTile;
    const int tps = (max_tiles + nsplit - 1) / nsplit;
    ri.tile0 = sp * tps;
    ri.tile1 = ri.tile0 + tps < ntiles ? ri.tile0 + tps : ntiles;
    if (!ri.ok) ri.tile1 = ri.tile0;
    return ri;
}

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void st_shared_b16(uint32_t addr, uint16_t v)
{
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__global__ void __launch_bounds__(kAttThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const int32_t *__restrict__ sel,
                   const int32_t *__restrict__ cu_q, const int32_t *__restrict__ cu_k, int batch,
                   int64_t row_begin, int64_t n_items, int nsplit, int kb, int r, float scale,
                   __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out,
                   float *__restrict__ ws)
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
        mbar_init(&sh->s_full, 1);
        mbar_init(&sh->o_full, 1);
        for (int i = 0; i < kNP; ++i) {
            mbar_init(&sh->p_full[i], 128);
            mbar_init(&sh->p_empty[i], 1);
        }
        sh->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sh->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    volatile int *abort_flag = &sh->abort_flag;

    if (warp == 0) {
        // ======================= TMA producer (whole warp) =======================
        if (lane == 0) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_k);
            tma_prefetch_desc(&map_v);
        }
        uint32_t slot_it = 0, q_it = 0;
        bool ok = true;
        for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const RowInfo ri = row_info(item, nsplit, row_begin, cu_q, cu_k, batch, kb, r);
            if (ri.tile0 >= ri.tile1) continue;
            if (lane == 0) {
                ok = mbar_wait(&sh->q_empty, (q_it & 1) ^ 1, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(&sh->q_full, kQBytes);
                    for (int g = 0; g < 2; ++g)
                        for (int c = 0; c < 4; ++c)
                            tma_load_2d(sQ + g * kQGroupBytes + c * 2048, &map_q, &sh->q_full, c * 64,
                                        (int32_t)(ri.row * kHQ + kGrp * g));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ++q_it;
            for (int g = 0; ok && g < 2; ++g) {
                for (int phase = 0; ok && phase < 2; ++phase) {
                    const CUtensorMap *map = phase == 0 ? &map_k : &map_v;
                    for (int j = ri.tile0; j < ri.tile1; ++j) {
                        const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
                        if (lane == 0) {
                            ok = mbar_wait(&sh->slot_empty[st], (round & 1) ^ 1, abort_flag);
                            if (ok) mbar_arrive_expect_tx(&sh->slot_full[st], kSlotBytes);
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        const int bi = j * kBlkPerTile + lane;
                        int32_t blk = bi < ri.nsel ? __ldg(sel + ri.row * kb + bi) : -1;
                        if (bi < ri.nsel && (blk < 0 || blk > ri.bt)) {
                            set_device_status(QSA_ERR_DEVICE_CHECK);
                            blk = -1;
                        }
                        const int32_t z = blk >= 0 ? (int32_t)(ri.tok_base + (int64_t)blk * r) : -4;
                        uint8_t *dst = sSlot + st * kSlotBytes + lane * 512;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_3d(dst + c * kChunk, map, &sh->slot_full[st], c * 64, g, z);
                        ++slot_it;
                    }
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
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 16, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 16, 1, 0);
            const uint32_t slot_addr = smem_u32(sSlot), q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            uint32_t slot_it = 0, q_it = 0, p_it = 0;
            bool ok = true;
            for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const RowInfo ri = row_info(item, nsplit, row_begin, cu_q, cu_k, batch, kb, r);
                if (ri.tile0 >= ri.tile1) continue;
                ok = mbar_wait(&sh->q_full, q_it & 1, abort_flag);
                ++q_it;
                for (int g = 0; ok && g < 2; ++g) {
                    // S^T tiles
                    for (int j = ri.tile0; ok && j < ri.tile1; ++j) {
                        const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
                        if (!(ok = mbar_wait(&sh->slot_full[st], round & 1, abort_flag))) break;
                        tc_fence_after();
                        const uint32_t a0 = slot_addr + st * kSlotBytes;
                        const uint32_t b0 = q_addr + g * kQGroupBytes;
                        const uint32_t d = tmem + kSCol + (j - ri.tile0) * 16;
#pragma unroll
                        for (int ks = 0; ks < kD / 16; ++ks) {
                            const uint32_t off = (ks & 3) * 32;
                            const uint64_t ad = sdesc_sw128(a0 + (ks >> 2) * kChunk + off, 16, 1024);
                            const uint64_t bd = sdesc_sw128(b0 + (ks >> 2) * 2048 + off, 16, 1024);
                            mma_bf16_ss(d, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(&sh->slot_empty[st]);
                        ++slot_it;
                    }
                    if (!ok) break;
                    if (g == 1) mma_commit(&sh->q_empty);
                    mma_commit(&sh->s_full);
                    // O^T += V^T P^T
                    for (int j = ri.tile0; ok && j < ri.tile1; ++j) {
                        const uint32_t st = slot_it % kNSlot, round = slot_it / kNSlot;
                        const uint32_t pb = p_it % kNP, pround = p_it / kNP;
                        if (!(ok = mbar_wait(&sh->slot_full[st], round & 1, abort_flag))) break;
                        if (!(ok = mbar_wait(&sh->p_full[pb], pround & 1, abort_flag))) break;
                        tc_fence_after();
                        const uint32_t a0 = slot_addr + st * kSlotBytes;
                        const uint32_t b0 = p_addr + pb * kPBytes;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const uint32_t d = tmem + kOCol + g * 32 + half * 16;
#pragma unroll
                            for (int ks = 0; ks < kTileTok / 16; ++ks) {
                                const uint64_t ad = sdesc_sw128(a0 + (2 * half) * kChunk + ks * 2048, kChunk, 1024);
                                const uint64_t bd = sdesc_sw128(b0 + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024);
                                mma_bf16_ss(d, ad, bd, idesc_pv, (j > ri.tile0 || ks > 0) ? 1u : 0u);
                            }
                        }
                        mma_commit(&sh->slot_empty[st]);
                        mma_commit(&sh->p_empty[pb]);
                        ++slot_it;
                        ++p_it;
                    }
                    if (!ok) break;
                    mma_commit(&sh->o_full);
                }
            }
        }
    } else {
        // ======================= softmax + epilogue (warps 2..5) =======================
        const int quad = warp & 3;
        const int key = quad * 32 + lane;           // TMEM lane = key within a tile
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const float c2 = scale * 1.4426950408889634f;
        const uint32_t p_addr = smem_u32(sP);
        const int kc64 = key & 63;
        const uint32_t p_key_off = (key >> 6) * 2048 + (kc64 & 7) * 2;
        const int p_unit = kc64 >> 3;
        uint32_t p_it = 0, grp_it = 0;
        bool ok = true;
        for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const RowInfo ri = row_info(item, nsplit, row_begin, cu_q, cu_k, batch, kb, r);
            const int sp = (int)(item % nsplit);
            const int64_t row_local = item / nsplit;
            if (ri.tile0 >= ri.tile1) {
                if (nsplit > 1) {  // empty split: neutral partial state
                    float *part = ws + ((row_local * nsplit + sp) * kHQ) * kD;
                    for (int x = key; x < kHQ * kD; x += 128) part[x] = 0.f;
                    float *lp = ws + (size_t)n_items * kHQ * kD + (row_local * nsplit + sp) * kHQ;
                    if (key < kHQ) lp[key] = -INFINITY;
                }
                continue;
            }
            // key validity per tile (bit j - tile0): selected block present, token <= t
            uint32_t vmask = 0;
            for (int j = ri.tile0; j < ri.tile1; ++j) {
                const int bi = j * kBlkPerTile + (key >> 2);
                if (bi < ri.nsel) {
                    const int32_t blk = __ldg(sel + ri.row * kb + bi);
                    const int64_t tok = (int64_t)blk * r + (key & 3);
                    if (blk >= 0 && blk <= ri.bt && tok <= ri.t) vmask |= 1u << (j - ri.tile0);
                }
            }
            const int nt = ri.tile1 - ri.tile0;
            for (int g = 0; ok && g < 2; ++g) {
                if (!(ok = mbar_wait(&sh->s_full, grp_it & 1, abort_flag))) break;
                tc_fence_after();
                float m[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) m[h] = -INFINITY;
                for (int jl = 0; jl < nt; ++jl) {
                    float s[16];
                    tmem_ld16(tmem + lane_addr + kSCol + jl * 16, s);
                    tmem_wait_ld();
                    if (vmask & (1u << jl)) {
#pragma unroll
                        for (int h = 0; h < 16; ++h) m[h] = fmaxf(m[h], s[h]);
                    }
                }
#pragma unroll
                for (int h = 0; h < 16; ++h) {
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
                }
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < 16; ++h) sh->red_max[quad][h] = m[h];
                }
                softmax_bar();
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    float x = fmaxf(fmaxf(sh->red_max[0][h], sh->red_max[1][h]), fmaxf(sh->red_max[2][h], sh->red_max[3][h]));
                    m[h] = (x == -INFINITY) ? 0.f : x;
                }
                float l[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) l[h] = 0.f;
                for (int jl = 0; ok && jl < nt; ++jl) {
                    const uint32_t pb = p_it % kNP, pround = p_it / kNP;
                    if (!(ok = mbar_wait(&sh->p_empty[pb], (pround & 1) ^ 1, abort_flag))) break;
                    float s[16];
                    tmem_ld16(tmem + lane_addr + kSCol + jl * 16, s);
                    tmem_wait_ld();
                    const bool valid = vmask & (1u << jl);
                    const uint32_t pbase = p_addr + pb * kPBytes + p_key_off;
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        const float p = valid ? exp2f((s[h] - m[h]) * c2) : 0.f;
                        l[h] += p;
                        const uint32_t addr = pbase + (h >> 3) * 1024 + (h & 7) * 128 + ((p_unit ^ (h & 7)) << 4);
                        st_shared_b16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(p)));
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(&sh->p_full[pb]);
                    ++p_it;
                }
                if (!ok) break;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
                }
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < 16; ++h) sh->red_sum[quad][h] = l[h];
                }
                softmax_bar();
                float inv[16];
                float my_lse = 0.f;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    const float L = sh->red_sum[0][h] + sh->red_sum[1][h] + sh->red_sum[2][h] + sh->red_sum[3][h];
                    inv[h] = L > 0.f ? 1.f / L : 0.f;
                    if (key == h) my_lse = m[h] * scale + logf(L);
                }
                if (!(ok = mbar_wait(&sh->o_full, grp_it & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[16];
                    tmem_ld16(tmem + lane_addr + kOCol + g * 32 + half * 16, o);
                    tmem_wait_ld();
                    const int d = half * 128 + key;
                    if (nsplit == 1) {
                        __nv_bfloat16 *dst = out + (ri.row * kHQ + g * kGrp) * kD + d;
#pragma unroll
                        for (int h = 0; h < kGrp; ++h) dst[h * kD] = __float2bfloat16_rn(o[h] * inv[h]);
                    } else {
                        float *dst = ws + ((row_local * nsplit + sp) * kHQ + g * kGrp) * kD + d;
#pragma unroll
                        for (int h = 0; h < kGrp; ++h) dst[h * kD] = o[h] * inv[h];
                    }
                }
                if (key < kGrp) {
                    if (nsplit == 1) {
                        if (lse_out != nullptr) lse_out[ri.row * kHQ + g * kGrp + key] = my_lse;
                    } else {
                        float *lp = ws + (size_t)n_items * kHQ * kD + (row_local * nsplit + sp) * kHQ;
                        lp[g * kGrp + key] = my_lse;
                    }
                }
                tc_fence_before();
                softmax_bar();  // red_* reuse by the next group
                ++grp_it;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// merge split-K partials: lse = logsumexp_s lse_s, o = sum_s exp(lse_s - lse) o_s
__global__ void __launch_bounds__(256)
combine_kernel(const float *__restrict__ ws, int64_t n_items, int nsplit, __nv_bfloat16 *__restrict__ out,
               float *__restrict__ lse_out)
{
    const int64_t row = blockIdx.x;
    const int h = blockIdx.y;
    const int d = threadIdx.x;
    const float *lp = ws + (size_t)n_items * kHQ * kD + row * nsplit * kHQ + h;
    float mx = -INFINITY;
    for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, lp[s * kHQ]);
    float tot = 0.f, acc = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float l = lp[s * kHQ];
        const float wgt = (l == -INFINITY) ? 0.f : __expf(l - mx);
        tot += wgt;
        acc += wgt * ws[((row * nsplit + s) * kHQ + h) * kD + d];
    }
    out[(row * kHQ + h) * kD + d] = __float2bfloat16_rn(tot > 0.f ? acc / tot : 0.f);
    if (lse_out != nullptr && d == 0) lse_out[row * kHQ + h] = mx + logf(tot);
}

}  // namespace

int min_nsplit(int kb)
{
    const int max_tiles = (kb + kBlkPerTile - 1) / kBlkPerTile;
    return (max_tiles + kMaxTiles - 1) / kMaxTiles;  // a split holds at most kMaxTiles tiles
}

int decode_nsplit(int batch, int kb)
{
    const int max_tiles = (kb + kBlkPerTile - 1) / kBlkPerTile;
    int ns = min_nsplit(kb);
    const int target = 2 * num_sms();
    while (ns * 2 <= max_tiles && (int64_t)batch * ns < target) ns *= 2;
    return ns;
}

size_t split_workspace_bytes(int64_t rows, int nsplit)
{
    return nsplit > 1 ? (size_t)rows * nsplit * kHQ * (kD + 1) * sizeof(float) : 0;
}

cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream)
{
    const int64_t rows = a.row_end - a.row_begin;
    if (rows <= 0) return cudaSuccess;
    CUtensorMap mq, mk, mv;
    // q as [rows_total * 24, 256]; k, v as [total_k][2][256] with a 64 x 1 x 4 box
    if (!make_tmap_2d(&mq, a.q, kD, (uint64_t)a.total_q * kHQ, kD * 2, 64, 16)) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mk, a.k, kD, kHKV, (uint64_t)a.total_k, kD * 2, kHKV * kD * 2, 64, 1, 4))
        return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mv, a.v, kD, kHKV, (uint64_t)a.total_k, kD * 2, kHKV * kD * 2, 64, 1, 4))
        return cudaErrorInvalidValue;
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
        attr = true;
    }
    const int max_tiles = (a.kb + kBlkPerTile - 1) / kBlkPerTile;
    if ((max_tiles + a.nsplit - 1) / a.nsplit > kMaxTiles) return cudaErrorInvalidValue;
    if (a.nsplit > 1 && a.ws == nullptr) return cudaErrorInvalidValue;
    const int64_t n_items = rows * a.nsplit;
    int64_t grid = num_sms();
    if (grid > n_items) grid = n_items;
    sparse_attn_kernel<<<(unsigned)grid, kAttThreads, kAttSmem, stream>>>(
        mq, mk, mv, a.sel, a.cu_q, a.cu_k, a.batch, a.row_begin, n_items, a.nsplit, a.kb, a.r, a.scale,
        a.o, a.lse, a.ws);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.nsplit == 1) return e;
    dim3 cg((unsigned)rows, kHQ);
    combine_kernel<<<cg, kD, 0, stream>>>(a.ws, n_items, a.nsplit, a.o + a.row_begin * kHQ * kD,
                                          a.lse ? a.lse + a.row_begin * kHQ : nullptr);
    return cudaGetLastError();
}

}  // namespace qsa
