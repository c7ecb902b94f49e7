// dense.cu -- dense causal GQA attention, the baseline the pages measure QSA
// against ("On the Design of Qwen3.8 Next Architecture", reading notes, result
// 2: kernel-level prefill and decode latency of QSA versus dense attention).
// Query t of a sequence attends to every key j <= t; head h reads KV group
// h / 12 (24 query heads, 2 KV heads, head dim 256, "Model Summary" table).
//
// Flash-attention forward on the 5th-generation tensor cores: one CTA per
// (128-query tile, head), heaviest (latest) tiles first.
//   warp 0      TMA producer: Q once, then 64-key K and V tiles (double-buffered)
//   warp 1      TMEM owner + single-thread MMA issue:
//                 S = Q K^T   M128 N64  K256  (K-major A and B), S double-buffered
//                 O += P V    M128 N256 K64   (P K-major from smem, V MN-major)
//   warps 2..5  softmax, thread = query row: row max and sum need no cross-thread
//               reduction; lazy rescale of the row's O in TMEM when the max grows
//               by more than 2^8; epilogue O / l -> bf16 and the log-sum-exp.
// TMEM: S 2 x 64 columns + O 256 columns.  Shared memory: Q 64 KB, K 2 x 32 KB,
// V 2 x 32 KB, P 2 x 16 KB.
#include "kernels.cuh"

namespace qsa {

namespace {

constexpr int kHQ = 24, kHKV = 2, kD = 256, kGrp = kHQ / kHKV;
constexpr int kBQ = 128;                     // queries per tile
constexpr int kBK = 64;                      // keys per tile
constexpr int kQChunk = kBQ * 128;           // 16 KB: 64 d-columns of the Q tile
constexpr int kQBytes = 4 * kQChunk;         // 64 KB
constexpr int kKChunk = kBK * 128;           // 8 KB
constexpr int kKVBytes = 4 * kKChunk;        // 32 KB per K or V tile
constexpr int kPBytes = kBQ * kBK * 2;       // 16 KB: P tile, one 64-key swizzled chunk
constexpr int kDenseThreads = 192;
constexpr uint32_t kSCol = 0, kOCol = 256, kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;

struct DenseShared {
    uint64_t q_full;
    uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2], p_empty[2];
    uint64_t o_full;  // every PV of the tile has completed
    uint32_t tmem_base;
    int abort_flag;
};

constexpr int kOffK = kQBytes;
constexpr int kOffV = kOffK + 2 * kKVBytes;
constexpr int kOffP = kOffV + 2 * kKVBytes;
constexpr int kOffSh = kOffP + 2 * kPBytes;
constexpr int kDenseSmem = kOffSh + (int)sizeof(DenseShared) + 1024;

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

struct TileInfo {
    int s;            // sequence
    int64_t q0;       // first packed query row of the tile
    int nq;           // valid queries in the tile
    int64_t k0;       // first packed key row of the sequence
    int64_t pos0;     // position of the tile's first query
    int nkt;          // key tiles to visit (causal)
    int64_t Lk;
    bool ok;
};

// Grid: blockIdx.x = tile slot (heaviest first), blockIdx.y = head.  Tiles of a
// sequence are 128-query blocks; tile ids run over the sequences in order.
__device__ __forceinline__ TileInfo tile_info(const int32_t *cu_q, const int32_t *cu_k, int batch,
                                              int ntiles_bound, int slot)
{
    TileInfo ti;
    ti.ok = false;
    ti.nkt = 0;
    const int tile = ntiles_bound - 1 - slot;
    int acc = 0, s = 0;
    for (; s < batch; ++s) {  // short walk: tiles per sequence = ceil(L_q / 128)
        const int nt = (cu_q[s + 1] - cu_q[s] + kBQ - 1) / kBQ;
        if (tile < acc + nt) break;
        acc += nt;
    }
    if (s >= batch) return ti;
    const int lt = tile - acc;
    ti.s = s;
    const int64_t Lq = (int64_t)cu_q[s + 1] - cu_q[s];
    ti.Lk = (int64_t)cu_k[s + 1] - cu_k[s];
    ti.q0 = cu_q[s] + (int64_t)lt * kBQ;
    ti.nq = (int)(Lq - (int64_t)lt * kBQ < kBQ ? Lq - (int64_t)lt * kBQ : kBQ);
    ti.k0 = cu_k[s];
    ti.pos0 = (ti.Lk - Lq) + (int64_t)lt * kBQ;
    ti.ok = ti.nq > 0 && ti.pos0 >= 0;
    ti.nkt = ti.ok ? (int)((ti.pos0 + ti.nq - 1) / kBK + 1) : 0;
    return ti;
}

__global__ void __launch_bounds__(kDenseThreads, 1)
dense_attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const int32_t *__restrict__ cu_q,
                  const int32_t *__restrict__ cu_k, int batch, int ntiles_bound, float scale,
                  __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = smem + kOffK;
    uint8_t *sV = smem + kOffV;
    uint8_t *sP = smem + kOffP;
    DenseShared *sh = reinterpret_cast<DenseShared *>(smem + kOffSh);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.y;
    const int g = head / kGrp;
    const TileInfo ti = tile_info(cu_q, cu_k, batch, ntiles_bound, blockIdx.x);
    if (!ti.ok) return;  // uniform for the CTA
    const int nkt = ti.nkt;

    if (threadIdx.x == 0) {
        mbar_init(&sh->q_full, 1);
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
        mbar_init(&sh->o_full, 1);
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
        // ---------------- TMA producer ----------------
        if (elect_one()) {
            tma_prefetch_desc(&map_q);
            tma_prefetch_desc(&map_k);
            tma_prefetch_desc(&map_v);
            mbar_arrive_expect_tx(&sh->q_full, kQBytes);
            for (int c = 0; c < 4; ++c)
                tma_load_3d(sQ + c * kQChunk, &map_q, &sh->q_full, c * 64, head, (int32_t)ti.q0);
            bool ok = true;
            // order: K0, V0, K1, V1, ... (each with its own double buffer)
            for (int j = 0; ok && j < nkt; ++j) {
                const uint32_t b = j & 1, rd = j >> 1;
                const int32_t krow = (int32_t)(ti.k0 + (int64_t)j * kBK);
                if (!(ok = mbar_wait(&sh->k_empty[b], (rd & 1) ^ 1, abort_flag))) break;
                mbar_arrive_expect_tx(&sh->k_full[b], kKVBytes);
                for (int c = 0; c < 4; ++c)
                    tma_load_3d(sK + b * kKVBytes + c * kKChunk, &map_k, &sh->k_full[b], c * 64, g, krow);
                if (!(ok = mbar_wait(&sh->v_empty[b], (rd & 1) ^ 1, abort_flag))) break;
                mbar_arrive_expect_tx(&sh->v_full[b], kKVBytes);
                for (int c = 0; c < 4; ++c)
                    tma_load_3d(sV + b * kKVBytes + c * kKChunk, &map_v, &sh->v_full[b], c * 64, g, krow);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (elect_one()) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBQ, kBK, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(kBQ, kD, 0, 1);
            const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV), p_addr = smem_u32(sP);
            bool ok = mbar_wait(&sh->q_full, 0, abort_flag);
            auto do_pv = [&](int j) -> bool {
                const uint32_t b = j & 1, rd = j >> 1;
                if (!mbar_wait(&sh->v_full[b], rd & 1, abort_flag)) return false;
                if (!mbar_wait(&sh->p_full[b], rd & 1, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kBK / 16; ++ks) {
                    // A = P (K-major, one 64-key chunk), B = V (MN-major: 64-d runs at LBO 8 KB, 8 keys at SBO 1 KB)
                    const uint64_t ad = sdesc_sw128(p_addr + b * kPBytes + ks * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(v_addr + b * kKVBytes + ks * 2048, kKChunk, 1024);
                    mma_bf16_ss(tmem + kOCol, ad, bd, idesc_pv, (j == 0 && ks == 0) ? 0u : 1u);
                }
                mma_commit(&sh->v_empty[b]);
                mma_commit(&sh->p_empty[b]);
                return true;
            };
            for (int j = 0; ok && j < nkt; ++j) {
                const uint32_t b = j & 1, rd = j >> 1;
                if (!(ok = mbar_wait(&sh->k_full[b], rd & 1, abort_flag))) break;
                if (!(ok = mbar_wait(&sh->s_empty[b], (rd & 1) ^ 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kQChunk + (ks & 3) * 32;
                    const uint32_t koff = (ks >> 2) * kKChunk + (ks & 3) * 32;
                    const uint64_t ad = sdesc_sw128(q_addr + off, 16, 1024);
                    const uint64_t bd = sdesc_sw128(k_addr + b * kKVBytes + koff, 16, 1024);
                    mma_bf16_ss(tmem + kSCol + b * kBK, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(&sh->k_empty[b]);
                mma_commit(&sh->s_full[b]);
                if (j >= 1) ok = do_pv(j - 1);
            }
            if (ok && do_pv(nkt - 1)) mma_commit(&sh->o_full);
        }
    } else {
        // ---------------- softmax + epilogue (warps 2..5) ----------------
        const int quad = warp & 3;
        const int row = quad * 32 + lane;              // TMEM lane = query row of the tile
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const int64_t pos = ti.pos0 + row;             // this row's position
        const bool row_ok = row < ti.nq;
        const float c2 = scale * 1.4426950408889634f;
        const uint32_t p_row = smem_u32(sP) + row * 128;
        float m = 0.f, l = 0.f;
        bool ok = true;
        for (int j = 0; ok && j < nkt; ++j) {
            const uint32_t b = j & 1, rd = j >> 1;
            if (!(ok = mbar_wait(&sh->s_full[b], rd & 1, abort_flag))) break;
            tc_fence_after();
            float s[kBK];
            tmem_ld32(tmem + lane_addr + kSCol + b * kBK, s);
            tmem_ld32(tmem + lane_addr + kSCol + b * kBK + 32, s + 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sh->s_empty[b]);
            const int64_t kbase = (int64_t)j * kBK;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kBK; ++c) {
                const bool valid = row_ok && kbase + c <= pos;
                s[c] = valid ? s[c] : -INFINITY;
                mx = fmaxf(mx, s[c]);
            }
            if (j == 0) {
                m = mx == -INFINITY ? 0.f : mx;
            } else if (mx > m + kRescaleLog2 / c2) {
                // lazy rescale of this row's running sum and of O (after the previous PV)
                const float f = exp2f((m - mx) * c2);
                m = mx;
                l *= f;
                // the previous PV has completed once its P buffer's last use is released
                if (!(ok = mbar_wait(&sh->p_empty[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < kD / 32; ++c) {
                    float o[32];
                    tmem_ld32(tmem + lane_addr + kOCol + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= f;
                    tmem_st32(tmem + lane_addr + kOCol + c * 32, o);
                }
                tmem_wait_st();
            }
            if (!(ok = mbar_wait(&sh->p_empty[b], (rd & 1) ^ 1, abort_flag))) break;
            // P row -> swizzled K-major tile: 64 keys = 8 units of 16 B, unit u at u ^ (row & 7)
            const uint32_t prow = p_row + b * kPBytes;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[e] = exp2f((s[u * 8 + e] - m) * c2);
                    l += p[e];
                }
                __nv_bfloat162 h0 = __floats2bfloat162_rn(p[0], p[1]), h1 = __floats2bfloat162_rn(p[2], p[3]);
                __nv_bfloat162 h2 = __floats2bfloat162_rn(p[4], p[5]), h3 = __floats2bfloat162_rn(p[6], p[7]);
                uint4 pk;
                pk.x = *reinterpret_cast<uint32_t *>(&h0);
                pk.y = *reinterpret_cast<uint32_t *>(&h1);
                pk.z = *reinterpret_cast<uint32_t *>(&h2);
                pk.w = *reinterpret_cast<uint32_t *>(&h3);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                             ::"r"(prow + ((u ^ (row & 7)) << 4)), "r"(pk.x), "r"(pk.y), "r"(pk.z), "r"(pk.w)
                             : "memory");
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&sh->p_full[b]);
        }
        if (ok) ok = mbar_wait(&sh->o_full, 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst = out + ((ti.q0 + row) * kHQ + head) * kD;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                float o[32];
                tmem_ld32(tmem + lane_addr + kOCol + c * 32, o);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(o[e] * inv, o[e + 1] * inv);
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(o[e + 2] * inv, o[e + 3] * inv);
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(o[e + 4] * inv, o[e + 5] * inv);
                        __nv_bfloat162 h3 = __floats2bfloat162_rn(o[e + 6] * inv, o[e + 7] * inv);
                        uint4 pk;
                        pk.x = *reinterpret_cast<uint32_t *>(&h0);
                        pk.y = *reinterpret_cast<uint32_t *>(&h1);
                        pk.z = *reinterpret_cast<uint32_t *>(&h2);
                        pk.w = *reinterpret_cast<uint32_t *>(&h3);
                        *reinterpret_cast<uint4 *>(dst + c * 32 + e) = pk;
                    }
                }
            }
            if (row_ok && lse_out != nullptr) lse_out[(ti.q0 + row) * kHQ + head] = m * scale + logf(l);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_dense_attn(const DenseArgs &a, cudaStream_t stream)
{
    if (a.total_q <= 0) return cudaSuccess;
    CUtensorMap mq, mk, mv;
    // q as (256 d, 24 heads, tokens), k and v as (256 d, 2 heads, tokens): 64 x 1 x rows boxes
    if (!make_tmap_3d(&mq, a.q, kD, kHQ, (uint64_t)a.total_q, kD * 2, (uint64_t)kHQ * kD * 2, 64, 1, kBQ))
        return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mk, a.k, kD, kHKV, (uint64_t)a.total_k, kD * 2, (uint64_t)kHKV * kD * 2, 64, 1, kBK))
        return cudaErrorInvalidValue;
    if (!make_tmap_3d(&mv, a.v, kD, kHKV, (uint64_t)a.total_k, kD * 2, (uint64_t)kHKV * kD * 2, 64, 1, kBK))
        return cudaErrorInvalidValue;
    {
        const cudaError_t e = set_smem_attr_once(reinterpret_cast<const void *>(dense_attn_kernel), kDenseSmem);
        if (e != cudaSuccess) return e;
    }
    // upper bound on tiles: every sequence may add one partial tile
    const int64_t max_tiles = (a.total_q + kBQ - 1) / kBQ + a.batch;
    dim3 grid((unsigned)max_tiles, kHQ);
    dense_attn_kernel<<<grid, kDenseThreads, kDenseSmem, stream>>>(mq, mk, mv, a.cu_q, a.cu_k, a.batch,
                                                                   (int)max_tiles, a.scale, a.o, a.lse);
    return cudaGetLastError();
}

}  // namespace qsa
