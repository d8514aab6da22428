// Chunked-prefill attention over the paged cache on tcgen05 tensor cores.
//
// What it computes ("vLLM — PagedAttention and Continuous Batching",
// s-samarth.github.io, §5 "Chunked prefill"; "How vLLM Works?", peterindia.net,
// §04): a sequence with context length c gets a chunk of q_len new query tokens
// at offset o = c - q_len. Chunk token j sits at position o + j and attends
// causally to keys 0 .. o + j of its paged context:
//   out[j][h] = softmax_k(scale * q[j][h] . K[k]) V[k],  k <= o + j,
// with K/V rows found through the block table, as in decode.
//
// How it runs (bf16 in, fp32 accumulate, head_dim 128):
//  * A CTA owns 128 rows = (128 / G) chunk tokens x the G query heads of one KV
//    head (GQA packing), so every K/V tile loaded serves all G heads.
//  * Q (128 x 128) and each K/V tile (128 keys x 128) come in by TMA with
//    128-byte swizzle. A K/V tile is eight 16-token blocks; each block of each
//    64-column half is one TMA box addressed through the block table. Blocks
//    past the context (and bad table entries) load from an out-of-range
//    coordinate, which fills zeros.
//  * S = Q K^T and O += P V run on the tensor cores (tcgen05.mma kind::f16,
//    M=128, N=128, K=16 per instruction) with accumulators in tensor memory:
//    two S buffers and one O, 384 of the 512 columns. QK of tile j+1 is issued
//    before the softmax of tile j, so the two overlap.
//  * Softmax: 8 warps. The two warps that share a TMEM lane quarter split each
//    row into 64-column halves and exchange partial maxima and sums through
//    shared memory. They mask keys past the row's causal limit and keep a
//    running max in the exp2 domain, with tree-shaped max/sum reductions. P goes
//    as bf16 into shared memory in the 128-byte-swizzled K-major layout the MMA
//    reads. O is rescaled in TMEM only when the row max grows by more than
//    2^8; otherwise the older max is kept, and P stays below 256.
//  * One thread issues the MMAs and commits them to mbarriers. Warp 0's lanes
//    0..7 issue the TMA loads, one block each. The table entries for a tile are
//    fetched one iteration before its loads.
//  * Every mbarrier wait is bounded. On a timeout the CTA flags
//    PA_STATUS_WAIT_TIMEOUT, waits (bounded) for its in-flight MMAs, frees its
//    tensor memory and returns.
#pragma once

#include <math_constants.h>

#include "pa_common.cuh"
#include "tmap.cuh"

namespace pa {

// ---- tcgen05 helpers ----------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc], bf16 x bf16 -> fp32, one thread issues.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes 32w..32w+31).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
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
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (sm_100 format):
// start address and the two byte offsets in 16-byte units, version 1, layout 2.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
    d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, A K-major,
// B K-major (b_mn = 0) or MN-major (b_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---- geometry -------------------------------------------------------------------

constexpr int kPfThreads = 256;
constexpr int kPfM = 128;  // rows per CTA
constexpr int kPfN = 128;  // keys per tile
constexpr int kPfD = 128;  // head_dim
constexpr int kPfHalf = kPfM * 64 * 2;          // one 64-column half of a 128-row bf16 tile: 16 KB
constexpr int kPfTile = 2 * kPfHalf;            // a 128 x 128 bf16 tile: 32 KB
constexpr int kPfOffQ = 0;
constexpr int kPfOffK = kPfOffQ + kPfTile;      // 2 stages
constexpr int kPfOffV = kPfOffK + 2 * kPfTile;  // 2 stages
constexpr int kPfOffP = kPfOffV + 2 * kPfTile;
constexpr int kPfOffBar = kPfOffP + kPfTile;    // mbarriers (8 B each)
constexpr int kPfBars = 9;                      // q, k[2], v[2], s[2], o, spare
constexpr int kPfOffSlot = kPfOffBar + kPfBars * 8;
constexpr int kPfOffRed = kPfOffSlot + 16;      // [2][128] floats: row max / row sum halves
constexpr int kPfSmem = kPfOffRed + 2 * 128 * 4 + 1024;  // + room to align the base to 1024 B
constexpr uint32_t kPfTmemCols = 512;
constexpr int kPfBlocksPerTile = kPfN / kBlockSize;
static_assert(kPfSmem <= 232448, "prefill shared memory over the 227 KB limit");
static_assert(kPfBlocksPerTile == 8, "warp 0 lanes 0..7 own one block each");

struct PrefillParams {
    void *out;
    const int *block_tables;
    const int *cu_q_lens;
    const int *context_lens;
    long long num_blocks;
    int max_blocks_per_seq;
    int num_heads;
    int num_kv_heads;
    int num_q_tokens;
    float scale_log2;
};

template <int G>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const PrefillParams prm, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    constexpr int TOK = kPfM / G;  // chunk tokens per CTA
    const int b = blockIdx.z, hk = blockIdx.y;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    // ---- per-sequence geometry (uniform over the CTA) ----
    const int q0 = __ldg(prm.cu_q_lens + b), q1 = __ldg(prm.cu_q_lens + b + 1);
    const int q_len = q1 - q0;
    const int c = __ldg(prm.context_lens + b);
    const bool first = blockIdx.x == 0 && hk == 0 && tid == 0;
    if (q_len < 0 || q_len > c || q1 > prm.num_q_tokens) {
        if (first) flag_status(PA_STATUS_BAD_QUERY);
        return;
    }
    if (c > prm.max_blocks_per_seq * kBlockSize) {
        if (first) flag_status(PA_STATUS_BAD_CONTEXT);
        return;
    }
    const int n_qt = (q_len + TOK - 1) / TOK;
    const int qt = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);  // longest tiles launch first
    if (qt >= n_qt) return;
    const int t0 = qt * TOK;
    const int o = c - q_len;
    const int rows_valid = min(TOK, q_len - t0);       // chunk tokens of this CTA
    const int kv_end = o + t0 + rows_valid;            // keys needed: [0, kv_end)
    const int n_tiles = (kv_end + kPfN - 1) / kPfN;
    const int nblk_seq = (c + kBlockSize - 1) / kBlockSize;

    // ---- shared memory (base aligned to 1024 B for the 128-byte swizzle) ----
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    unsigned char *base = smem_raw + (base_s - raw_s);
    const uint32_t sQ = base_s + kPfOffQ, sK = base_s + kPfOffK, sV = base_s + kPfOffV, sP = base_s + kPfOffP;
    const uint32_t bar_q = base_s + kPfOffBar;
    const uint32_t bar_k = bar_q + 8;       // [2]
    const uint32_t bar_v = bar_q + 24;      // [2]
    const uint32_t bar_s = bar_q + 40;      // [2]
    const uint32_t bar_o = bar_q + 56;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kPfOffSlot);

    if (tid == 0) {
        mbar_init(bar_q, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_k + 8 * i, 1);
            mbar_init(bar_v + 8 * i, 1);
            mbar_init(bar_s + 8 * i, 1);
        }
        mbar_init(bar_o, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(smem_addr(tmem_slot), kPfTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tO = tmem + 256;  // S tiles at columns 0 and 128

    // ---- loads (warp 0) ----
    const int *trow = prm.block_tables + static_cast<size_t>(b) * prm.max_blocks_per_seq;
    const int oob_row = static_cast<int>(prm.num_blocks * kBlockSize);  // a row past the pool: TMA fills zeros
    // pool row of block `lane` (0..7) of tile t, or the out-of-range row
    auto tile_row = [&](int t) -> int {
        if (lane >= kPfBlocksPerTile) return oob_row;
        const int lb = t * kPfBlocksPerTile + lane;
        if (t >= n_tiles || lb >= nblk_seq) return oob_row;
        const int pb = __ldg(trow + lb);
        if (pb < 0 || pb >= prm.num_blocks) {
            flag_status(PA_STATUS_BAD_BLOCK_ID);
            return oob_row;
        }
        return pb * kBlockSize;
    };
    auto load_tile = [&](const CUtensorMap *tm, uint32_t dst, uint32_t bar, int row) {
        if (lane == 0) mbar_arrive_expect_tx(bar, kPfTile);
        __syncwarp();
        if (lane < kPfBlocksPerTile) {
            const uint32_t d = dst + lane * (kBlockSize * 128);  // 16 rows of 128 B
            tma_load_3d(d, tm, 0, hk, row, bar);
            tma_load_3d(d + kPfHalf, tm, 64, hk, row, bar);
        }
    };
    int row_a = 0, row_b = 0, row_c = 0;  // warp 0: pool rows of tiles j+1, j+2, j+3 (row_a = j+1)
    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(bar_q, kPfTile);
            const int qrow = q0 + t0;
            tma_load_3d(sQ, &tm_q, 0, hk * G, qrow, bar_q);
            tma_load_3d(sQ + kPfHalf, &tm_q, 64, hk * G, qrow, bar_q);
        }
        const int r0 = tile_row(0);
        row_a = tile_row(1);
        row_b = tile_row(2);
        load_tile(&tm_k, sK, bar_k, r0);
        load_tile(&tm_v, sV, bar_v, r0);
        if (n_tiles > 1) {
            load_tile(&tm_k, sK + kPfTile, bar_k + 8, row_a);
            load_tile(&tm_v, sV + kPfTile, bar_v + 8, row_a);
        }
        row_c = tile_row(3);
    }

    constexpr uint32_t kIdQK = idesc_bf16(kPfM, kPfN, 0);
    constexpr uint32_t kIdPV = idesc_bf16(kPfM, kPfD, 1);
    // S_t = Q K_t^T into tS[t % 2]
    auto issue_qk = [&](int t) {
        const uint32_t kb = sK + (t & 1) * kPfTile;
#pragma unroll
        for (int kk = 0; kk < kPfD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kPfHalf + (kk & 3) * 32;
            umma_bf16(tmem + (t & 1) * kPfN, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024), kIdQK,
                      kk > 0);
        }
        umma_commit(bar_s + 8 * (t & 1));
    };
    // O += P V_t
    auto issue_pv = [&](int t) {
        const uint32_t vb = sV + (t & 1) * kPfTile;
#pragma unroll
        for (int kk = 0; kk < kPfN / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * kPfHalf + (kk & 3) * 32;
            umma_bf16(tO, smem_desc_sw128(sP + aoff, 16, 1024), smem_desc_sw128(vb + kk * 2048, kPfHalf, 1024), kIdPV,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar_o);
    };

    bool ok = true;
    int qk_issued = 0;  // tid 0 only: QK tiles issued
    if (tid == 0) {
        ok = mbar_wait(bar_q, 0) && mbar_wait(bar_k, 0);
        if (ok) {
            tc_fence_after();
            issue_qk(0);
            qk_issued = 1;
        }
    }

    // ---- per-row state: warps w and w+4 share TMEM lanes 32(w%4).., and each takes
    // one 64-column half of the row (keys of the S tile, dims of O) ----
    const int quarter = warp & 3, hcol = warp >> 2;
    const int r = quarter * 32 + lane;
    const int tok = min(t0 + r / G, q_len - 1);  // rows past the chunk reuse the last token's limit
    const int pos = o + tok;                     // causal limit: keys 0..pos
    float m_ref = -CUDART_INF_F;                 // reference max (log2 domain) of the row
    float l_sum = 0.f;                           // this thread's half of the row sum
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    float *red = reinterpret_cast<float *>(base + kPfOffRed);  // [2][128] partial row max, then sums
    int pv_issued = 0;

    for (int j = 0; j < n_tiles; ++j) {
        // 1. S_j ready
        ok = __syncthreads_and(ok ? 1 : 0) != 0;
        if (!ok) break;
        bool w = mbar_wait(bar_s + 8 * (j & 1), (j >> 1) & 1);
        tc_fence_after();
        // 2. refill the K stage QK_j just read; issue QK_{j+1}
        if (warp == 0) {
            if (j + 2 < n_tiles) load_tile(&tm_k, sK + (j & 1) * kPfTile, bar_k + 8 * (j & 1), row_b);
            if (tid == 0 && j + 1 < n_tiles && w) {
                w = mbar_wait(bar_k + 8 * ((j + 1) & 1), ((j + 1) >> 1) & 1);
                if (w) {
                    tc_fence_after();
                    issue_qk(j + 1);
                    qk_issued = j + 2;
                }
            }
        }
        // 3. PV_{j-1} done: O stable, P buffer and V stage (j-1)&1 free
        if (j > 0) {
            w = mbar_wait(bar_o, (j - 1) & 1) && w;
            tc_fence_after();
            if (warp == 0 && j + 1 < n_tiles)
                load_tile(&tm_v, sV + ((j + 1) & 1) * kPfTile, bar_v + 8 * ((j + 1) & 1), row_a);
        }
        if (warp == 0) {  // advance the table window: rows of tiles j+2, j+3, j+4
            row_a = row_b;
            row_b = row_c;
            row_c = tile_row(j + 4);
        }
        // 4a. the tile's keys past the context: their V rows (tail slots of the
        // last block) may hold anything, and 0 * NaN would poison O, so zero them
        if ((j + 1) * kPfN > c) {
            w = mbar_wait(bar_v + 8 * (j & 1), (j >> 1) & 1) && w;
            const int first_bad = max(0, c - j * kPfN);
            const int n16 = (kPfN - first_bad) * 2 * 8;  // 16-byte chunks in both halves
            unsigned char *vt = base + kPfOffV + (j & 1) * kPfTile;
            for (int i = tid; i < n16; i += kPfThreads) {
                const int row = first_bad + i / 16, half = (i / 8) & 1, chunk = i & 7;
                *reinterpret_cast<uint4 *>(vt + half * kPfHalf + row * 128 + chunk * 16) = make_uint4(0, 0, 0, 0);
            }
        }
        __syncwarp();
        // 4b. this thread's 64 scores of row r
        constexpr int HN = kPfN / 2;
        float s[HN];
        const uint32_t s_cols = tmem + (j & 1) * kPfN + hcol * HN;
#pragma unroll
        for (int ch = 0; ch < HN / 32; ++ch) {
            float v[32];
            tmem_ld32(s_cols + lane_base + ch * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) s[ch * 32 + i] = v[i] * prm.scale_log2;
        }
        const int key0 = j * kPfN + hcol * HN;
        if (key0 + HN - 1 > pos) {
#pragma unroll
            for (int i = 0; i < HN; ++i)
                if (key0 + i > pos) s[i] = -CUDART_INF_F;
        }
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
        for (int i = 8; i < HN; ++i) m8[i & 7] = fmaxf(m8[i & 7], s[i]);
        const float mx_half = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                    fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        red[hcol * kPfM + r] = mx_half;
        __syncthreads();
        const float mx = fmaxf(red[r], red[kPfM + r]);
        float alpha = 1.f;
        if (mx > m_ref + 8.f || m_ref == -CUDART_INF_F) {
            const float m_new = fmaxf(mx, m_ref);
            alpha = (m_ref == -CUDART_INF_F) ? 0.f : exp2f(m_ref - m_new);
            m_ref = m_new;
        }
        float a8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a8[i] = 0.f;
        unsigned char *prow = base + kPfOffP + hcol * kPfHalf + r * 128;
#pragma unroll
        for (int cc = 0; cc < HN / 8; ++cc) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p0 = m_ref == -CUDART_INF_F ? 0.f : exp2f(s[cc * 8 + 2 * e] - m_ref);
                const float p1 = m_ref == -CUDART_INF_F ? 0.f : exp2f(s[cc * 8 + 2 * e + 1] - m_ref);
                const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                a8[(2 * e) & 7] += __low2float(pb);
                a8[(2 * e + 1) & 7] += __high2float(pb);
                pk[e] = *reinterpret_cast<const uint32_t *>(&pb);
            }
            *reinterpret_cast<uint4 *>(prow + ((cc ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        const float psum = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
        l_sum = l_sum * alpha + psum;
        // rescale this thread's half of O's row in tensor memory (warp-uniform:
        // tcgen05.ld/st are .sync.aligned)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int ch = 0; ch < HN / 32; ++ch) {
                const uint32_t oc = tO + hcol * HN + lane_base + ch * 32;
                float v[32];
                tmem_ld32(oc, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= alpha;
                tmem_st32(oc, v);
            }
        }
        // 5. P visible to the tensor core, TMEM reads/writes ordered before the next MMA
        fence_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(w ? 1 : 0) != 0;
        if (!ok) break;
        // 6. O += P V_j
        if (tid == 0) {
            tc_fence_after();
            if (mbar_wait(bar_v + 8 * (j & 1), (j >> 1) & 1)) {
                issue_pv(j);
            } else {
                ok = false;
            }
        }
        pv_issued = j + 1;
    }
    ok = __syncthreads_and(ok ? 1 : 0) != 0;

    // ---- epilogue: out = O / l for the valid rows, each thread its 64 dims ----
    if (ok && pv_issued == n_tiles && n_tiles > 0) {
        red[hcol * kPfM + r] = l_sum;
        ok = mbar_wait(bar_o, (n_tiles - 1) & 1);
        ok = __syncthreads_and(ok ? 1 : 0) != 0;
        tc_fence_after();
        if (ok) {
            const float l_row = red[r] + red[kPfM + r];
            const bool row_ok = r / G < rows_valid;
            const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
            const int orow = row_ok ? q0 + t0 + r / G : q0;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(prm.out) +
                                 (static_cast<size_t>(orow) * prm.num_heads + hk * G + r % G) * kPfD + hcol * 64;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                float v[32];
                tmem_ld32(tO + hcol * 64 + lane_base + ch * 32, v);
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    uint4 pkt;
                    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[i] * inv, v[i + 1] * inv);
                    __nv_bfloat162 h1 = __floats2bfloat162_rn(v[i + 2] * inv, v[i + 3] * inv);
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[i + 4] * inv, v[i + 5] * inv);
                    __nv_bfloat162 h3 = __floats2bfloat162_rn(v[i + 6] * inv, v[i + 7] * inv);
                    pkt.x = *reinterpret_cast<uint32_t *>(&h0);
                    pkt.y = *reinterpret_cast<uint32_t *>(&h1);
                    pkt.z = *reinterpret_cast<uint32_t *>(&h2);
                    pkt.w = *reinterpret_cast<uint32_t *>(&h3);
                    if (row_ok) *reinterpret_cast<uint4 *>(dst + ch * 32 + i) = pkt;
                }
            }
        }
    } else if (tid == 0) {
        // failed: let the MMAs already issued finish before tensor memory is freed
        if (pv_issued > 0) mbar_wait(bar_o, (pv_issued - 1) & 1);
        if (qk_issued > 0) mbar_wait(bar_s + 8 * ((qk_issued - 1) & 1), ((qk_issued - 1) >> 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

template <int G>
int launch_prefill_g(const PrefillParams &prm, const void *q, const void *k_cache, const void *v_cache,
                     int num_seqs, int max_q_len, int num_q_tokens, const pa_shape *s, cudaStream_t st) {
    constexpr int TOK = kPfM / G;
    CUtensorMap tm_q{}, tm_k{}, tm_v{};
    const uint64_t rows = static_cast<uint64_t>(s->num_blocks) * kBlockSize;
    if (!encode_3d(&tm_q, q, kPfD, s->num_heads, num_q_tokens, 2, 64, G, TOK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_3d(&tm_k, k_cache, kPfD, s->num_kv_heads, rows, 2, 64, 1, kBlockSize, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_3d(&tm_v, v_cache, kPfD, s->num_kv_heads, rows, 2, 64, 1, kBlockSize, CU_TENSOR_MAP_SWIZZLE_128B))
        return PA_ERR_UNSUPPORTED;
    static bool attr_done[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(prefill_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmem) !=
            cudaSuccess)
            return PA_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int n_qt = (max_q_len + TOK - 1) / TOK;
    const dim3 grid(n_qt, s->num_kv_heads, num_seqs);
    prefill_kernel<G><<<grid, kPfThreads, kPfSmem, st>>>(prm, tm_q, tm_k, tm_v);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

inline int launch_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *cu_q_lens,
                          const int32_t *context_lens, int32_t num_seqs, int32_t max_q_len, int32_t num_q_tokens,
                          float scale, const pa_shape *s, cudaStream_t st) {
    if (num_seqs > 65535 || s->num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    PrefillParams prm{};
    prm.out = out;
    prm.block_tables = block_tables;
    prm.cu_q_lens = cu_q_lens;
    prm.context_lens = context_lens;
    prm.num_blocks = s->num_blocks;
    prm.max_blocks_per_seq = max_blocks_per_seq;
    prm.num_heads = s->num_heads;
    prm.num_kv_heads = s->num_kv_heads;
    prm.num_q_tokens = num_q_tokens;
    prm.scale_log2 = scale * 1.4426950408889634f;
    switch (s->num_heads / s->num_kv_heads) {
        case 1: return launch_prefill_g<1>(prm, q, k_cache, v_cache, num_seqs, max_q_len, num_q_tokens, s, st);
        case 2: return launch_prefill_g<2>(prm, q, k_cache, v_cache, num_seqs, max_q_len, num_q_tokens, s, st);
        case 4: return launch_prefill_g<4>(prm, q, k_cache, v_cache, num_seqs, max_q_len, num_q_tokens, s, st);
        case 8: return launch_prefill_g<8>(prm, q, k_cache, v_cache, num_seqs, max_q_len, num_q_tokens, s, st);
        default: return PA_ERR_UNSUPPORTED;
    }
}

}  // namespace pa
