// Decode-time paged attention (one query token per sequence), sm_100a.
//
// What it computes ("vLLM and PagedAttention", ai.zenoagi.com, §2 "Reworking
// the Attention Computation"): for each sequence b and query head h,
//   out[b][h] = softmax(scale * q[b][h] . K_b^T) V_b
// where row p of K_b/V_b sits in physical block block_tables[b][p / 16] at row
// p % 16. Blocks are loaded one by one and each block's share is folded into
// a running result. That is online softmax: a running max m, a running sum l
// and an accumulator O rescaled by exp(m_old - m_new) whenever m grows.
//
// How it runs on B200:
//  * Grid (KV head, sequence, partition). A CTA owns one KV head of one
//    sequence over one partition of the context (split-context pass).
//    Sequences longer than a partition write (m, l, O) partials, and the last
//    CTA of the (sequence, KV head) to finish merges them (a ticket counter in
//    the workspace), so pa_decode is one kernel. The merge can also run as its
//    own kernel (decode_reduce_kernel), with the same arithmetic.
//  * Every query head of the KV head's group (G = H / Hk of them) reads each
//    loaded block from shared memory, so K/V cross HBM once per KV head.
//  * The 4 warps of a CTA take the partition's blocks round-robin. Each warp
//    streams its own blocks through an NSTAGE-deep shared-memory ring. A
//    block's 16 K rows and 16 V rows of one KV head are two TMA tiled loads
//    (a [16][D] box of the pool viewed as [NB*16][Hk][D]) into a ring slot,
//    and an mbarrier counts the bytes. Fetches run NSTAGE blocks ahead.
//  * Lanes own column slices of a row made of CH chunks of CB bytes,
//    interleaved so shared-memory reads are conflict free. L lanes cover a
//    row and RS = 32 / L rows are processed per step.
//  * q.k: each lane forms NPART = STEPS * G partial dot products per block,
//    and a transpose-reduce over the L lanes of a row halves the values per
//    lane at each shuffle step. Lanes visit the steps and hold the heads in a
//    lane-dependent order (an XOR of step and head indices by the lane's
//    column bits), chosen so that at every shuffle step each lane keeps its
//    first half and sends its second: no selects. A lane ends with NFIN
//    complete scores, one row and NFIN consecutive heads.
//  * Softmax in fp32 in the exp2 domain (scale * log2(e) folded into q). The
//    running max of a head moves (and O, l are rescaled) only when a score
//    exceeds it by more than 8, so the common block takes no reduction: each
//    lane exponentiates its own scores and stores them, duplicated as packed
//    pairs, in a small per-warp buffer that P.V reads back as broadcasts.
//  * P.V uses packed two-wide fp32 FMAs on (even, odd) column pairs.
//  * Each warp keeps its own (m, l, O). At the end the warps merge through
//    shared memory (reusing the ring).
#pragma once

#include <math_constants.h>

#include "pa_common.cuh"
#include "tmap.cuh"

namespace pa {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = 32 * kDecodeWarps;

template <typename T, int D, int G>
struct DecodeCfg {
    static constexpr int E = sizeof(T);
    static constexpr int R = D * E;                        // bytes of one token row of one KV head
    // Bytes of one chunk: 16, or 8 for FP8 rows with groups of 8 heads, so that
    // a lane holds 8 dims per row as for bf16 (16 would spill q and O).
    static constexpr int CB = (E == 1 && G >= 8) ? 8 : 16;
    static constexpr int CH = (G >= 8 || E == 1) ? 1 : 2;  // chunks a lane owns per row
    static constexpr int L = R / (CB * CH);                // lanes covering one row
    static constexpr int RS = 32 / L;                      // rows per warp step
    static constexpr int STEPS = kBlockSize / RS;          // steps per block
    static constexpr int VE = CB / E;                      // elements per chunk
    static constexpr int EPL = CH * VE;                    // elements per lane per row
    static constexpr int P2 = EPL / 2;                     // packed pairs per lane per row
    static constexpr int STAGE_BYTES = 2 * kBlockSize * R; // K and V of one block
    // Two stages per warp and three CTAs per SM (12 warps) measured faster on
    // B200 than three stages at two CTAs per SM.
#ifndef PA_DECODE_NSTAGE
#define PA_DECODE_NSTAGE 2
#endif
#ifndef PA_DECODE_PF
#define PA_DECODE_PF 0
#endif
    static constexpr int NSTAGE = PA_DECODE_NSTAGE;
    // Blocks ahead of the one being loaded into shared memory whose K and V
    // are prefetched into L2 (0: none).
    static constexpr int PF = PA_DECODE_PF;
    // CTAs per SM the register budget is sized for (wide rows keep more live state).
#ifndef PA_DECODE_MINB4
#define PA_DECODE_MINB4 3
#endif
    static constexpr int MIN_BLOCKS = G <= 4 ? PA_DECODE_MINB4 : 2;
    static constexpr int WARP_RING = NSTAGE * STAGE_BYTES;
    static constexpr int RING_BYTES = kDecodeWarps * WARP_RING;
    static constexpr int NPART = STEPS * G;                 // q.k partials per lane per block
    static constexpr int NFIN = NPART >= L ? NPART / L : 1; // complete scores per lane
    static constexpr int DUP = NPART >= L ? 1 : L / NPART;  // lanes holding the same scores
    static constexpr int PBUF = kBlockSize * G * 8;         // per warp: [16 rows][G heads] of (p, p)
    static constexpr int RED_BYTES = kDecodeWarps * RS * G * D * 4;
    static constexpr int BIG = RING_BYTES > RED_BYTES ? RING_BYTES : RED_BYTES;
    static constexpr int OFF_BAR = BIG;
    static constexpr int OFF_P = OFF_BAR + kDecodeWarps * NSTAGE * 8;
    static constexpr int OFF_ML = OFF_P + kDecodeWarps * PBUF;
    static constexpr int OFF_FLAG = OFF_ML + 2 * kDecodeWarps * G * 4;
    static constexpr int SMEM = OFF_FLAG + 16;
    static_assert(R % (CB * CH) == 0 && L >= 1 && L <= 32 && 32 % L == 0, "row must split into lane slices");
    static_assert(kBlockSize % RS == 0, "rows per step must divide the block");
    static_assert(32 % G == 0 && G <= 8, "group size");
    static_assert(G % NFIN == 0, "a lane's scores are consecutive heads of one row");
    static_assert(OFF_P % 16 == 0, "probability buffer alignment");
    static_assert(STEPS >= 2 && L >= 4, "the first reduce step pairs step slots s and s + STEPS / 2");
};

// Sum, over the lanes that differ in the bits OFF, OFF/2, ..., 1, the N values
// each lane holds. Each step adds the partner's second half to the lane's
// first half (v[i] += partner's v[i + N/2]). That is a transpose-reduce when
// the lane whose OFF bit is set holds its values with the halves swapped,
// which the callers arrange by the order in which they compute them. Once one
// value is left, the remaining steps are plain butterfly sums.
template <int N, int OFF>
struct TransposeReduce {
    template <int NA>
    __device__ __forceinline__ static void run(float (&v)[NA]) {
        if constexpr (OFF == 0) {
            return;
        } else if constexpr (N > 1) {
            constexpr int H = N / 2;
#pragma unroll
            for (int i = 0; i < H; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i + H], OFF);
            TransposeReduce<H, OFF / 2>::run(v);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
            TransposeReduce<1, OFF / 2>::run(v);
        }
    }
};

// Widen one CB-byte chunk of a cache row from shared memory to VE / 2 pairs.
template <typename T, int CB>
__device__ __forceinline__ void load_chunk(const unsigned char *p, f32x2 *f) {
    if constexpr (CB == 16) {
        Widen<T>::apply2(*reinterpret_cast<const uint4 *>(p), f);
    } else {
        static_assert(CB == 8 && sizeof(T) == 1, "8-byte chunks are for FP8 rows");
        const uint2 r = *reinterpret_cast<const uint2 *>(p);
        f[0] = e4m3x2_to_f32x2(r.x & 0xffffu);
        f[1] = e4m3x2_to_f32x2(r.x >> 16);
        f[2] = e4m3x2_to_f32x2(r.y & 0xffffu);
        f[3] = e4m3x2_to_f32x2(r.y >> 16);
    }
}

__device__ __forceinline__ void lds_pair2(uint32_t addr, f32x2 &a, f32x2 &b) {
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr) : "memory");
}

__device__ __forceinline__ f32x2 lds_pair(uint32_t addr) {
    f32x2 a;
    asm volatile("ld.shared.b64 %0, [%1];" : "=l"(a) : "r"(addr) : "memory");
    return a;
}

struct DecodeParams {
    void *out;
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int *block_tables;
    const int *context_lens;
    float *ws_o;  // [B][H][max_parts][D]
    float *ws_m;  // [B][H][max_parts]
    float *ws_l;  // [B][H][max_parts]
    unsigned long long *ws_ticket;  // [B][Hk] tickets of the fused merge: (call stamp << 32) | arrivals
    long long num_blocks;
    int max_blocks_per_seq;
    int num_heads;
    int num_kv_heads;
    int max_context_len;
    int part_tokens;
    int max_parts;
    int fuse_merge;    // 1: the last partition CTA of a unit merges; 0: decode_reduce_kernel does
    unsigned int stamp;  // nonzero, different for every host call: a ticket with another stamp counts as 0
    float scale_log2;  // softmax scale * log2(e) (times k_scale for an FP8 cache)
    float v_scale;     // 1, or the FP8 value scale
};

// Merge the `parts` partials of query head h of sequence b for column d:
//   M = max_p m_p,  L = sum_p 2^(m_p - M) l_p,  out = sum_p 2^(m_p - M) O_p / L,
// in one pass with a running max, loading up to 8 partitions at a time.
// The fused merge and decode_reduce_kernel share it, so both give the same bits.
template <typename T>
__device__ __forceinline__ void merge_partitions(const DecodeParams &prm, int b, int h, int parts, int d, int D) {
    const size_t base = (static_cast<size_t>(b) * prm.num_heads + h) * prm.max_parts;
    float M = -CUDART_INF_F, O = 0.f, L = 0.f;
    for (int p0 = 0; p0 < parts; p0 += 8) {
        float mp[8], lp[8], op[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool in = p0 + i < parts;
            mp[i] = in ? __ldcg(prm.ws_m + base + p0 + i) : -CUDART_INF_F;
            lp[i] = in ? __ldcg(prm.ws_l + base + p0 + i) : 0.f;
            op[i] = in ? __ldcg(prm.ws_o + (base + p0 + i) * D + d) : 0.f;
        }
        float mc = M;
#pragma unroll
        for (int i = 0; i < 8; ++i) mc = fmaxf(mc, mp[i]);
        if (mc == -CUDART_INF_F) continue;
        const float a = exp2f(M - mc);  // 0 while M is still -inf
        O *= a;
        L *= a;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float wt = mp[i] == -CUDART_INF_F ? 0.f : exp2f(mp[i] - mc);
            O += wt * op[i];
            L += wt * lp[i];
        }
        M = mc;
    }
    T *out = static_cast<T *>(prm.out) + (static_cast<size_t>(b) * prm.num_heads + h) * D + d;
    store_out(out, L > 0.f ? O / L : 0.f);
}

// merge_partitions for up to NE output elements of one (sequence, KV head)
// group at once, elements idx0 + e * stride (e < NE, below `total`) of its
// [G][D] outputs, with the loads of all of them in flight together. Per
// element, the arithmetic is merge_partitions' (the same bits).
template <typename T, int NE>
__device__ __forceinline__ void merge_partitions_n(const DecodeParams &prm, int b, int h0, int idx0, int stride,
                                                   int total, int parts, int D) {
    size_t base[NE];
    int dd[NE];
    float M[NE], O[NE], L[NE];
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        const int idx = min(idx0 + e * stride, total - 1);  // past the end: a copy of the last, not stored
        base[e] = (static_cast<size_t>(b) * prm.num_heads + h0 + idx / D) * prm.max_parts;
        dd[e] = idx % D;
        M[e] = -CUDART_INF_F;
        O[e] = 0.f;
        L[e] = 0.f;
    }
    for (int p0 = 0; p0 < parts; p0 += 8) {
        float mp[NE][8], lp[NE][8], op[NE][8];
#pragma unroll
        for (int e = 0; e < NE; ++e)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const bool in = p0 + i < parts;
                mp[e][i] = in ? __ldcg(prm.ws_m + base[e] + p0 + i) : -CUDART_INF_F;
                lp[e][i] = in ? __ldcg(prm.ws_l + base[e] + p0 + i) : 0.f;
                op[e][i] = in ? __ldcg(prm.ws_o + (base[e] + p0 + i) * D + dd[e]) : 0.f;
            }
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            float mc = M[e];
#pragma unroll
            for (int i = 0; i < 8; ++i) mc = fmaxf(mc, mp[e][i]);
            if (mc == -CUDART_INF_F) continue;
            const float a = exp2f(M[e] - mc);  // 0 while M is still -inf
            O[e] *= a;
            L[e] *= a;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float wt = mp[e][i] == -CUDART_INF_F ? 0.f : exp2f(mp[e][i] - mc);
                O[e] += wt * op[e][i];
                L[e] += wt * lp[e][i];
            }
            M[e] = mc;
        }
    }
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        const int idx = idx0 + e * stride;
        if (idx >= total) break;
        T *out = static_cast<T *>(prm.out) + (static_cast<size_t>(b) * prm.num_heads + h0 + idx / D) * D + dd[e];
        store_out(out, L[e] > 0.f ? O[e] / L[e] : 0.f);
    }
}

// Tq: element type of q and out. Tc: element type of the caches (the same, or
// FP8 E4M3 codes with bf16 q/out).
template <typename Tq, typename Tc, int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, DecodeCfg<Tc, D, G>::MIN_BLOCKS)
    decode_kernel(const DecodeParams prm, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v) {
    using C = DecodeCfg<Tc, D, G>;
    constexpr int P2 = C::P2;      // packed pairs per lane per row
    constexpr int VP = C::VE / 2;  // packed pairs per chunk
    // Grid (KV head, sequence, partition): every unit's first partition launches
    // before any second one, so full partitions run first and the short last
    // partitions (or empty CTAs) form the tail.
    const int hk = blockIdx.x, b = blockIdx.y, p = blockIdx.z;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int rg = lane / C::L, j = lane % C::L;

    // The lane's step and head order for the transpose-reduce: at the reduce
    // step whose partner differs in lane bit `off`, values i and i + h (h half
    // the values left) trade places in the lane with that bit set. Over all
    // steps, step slot s holds step s ^ smask and head slot g holds head
    // g ^ hmask. A lane ends with the scores of row smask * RS + rg, heads
    // hmask .. hmask + NFIN - 1.
    int smask = 0, hmask = 0;
    {
        int n = C::NPART;
#pragma unroll
        for (int off = C::L / 2; off >= 1; off >>= 1) {
            if (n >= 2) {
                const int h = n / 2;
                if (lane & off) {
                    if (h >= G) smask ^= h / G;
                    else hmask ^= h;
                }
                n = h;
            }
        }
    }

    // Launched as a programmatic dependent (its launch overlaps the previous
    // kernel, e.g. the cache write): wait for that kernel before reading any input.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int part_blocks = prm.part_tokens / kBlockSize;
    const int blk0 = p * part_blocks;
    const int *trow = prm.block_tables + static_cast<size_t>(b) * prm.max_blocks_per_seq + blk0;
    // The length and this warp's first table entries load together (the
    // entries are only used for blocks inside the context).
    const int c_raw = __ldg(prm.context_lens + b);
    const int tbl_lim = min(part_blocks, prm.max_blocks_per_seq - blk0);
    int tbl = 0;
    if (warp + lane * kDecodeWarps < tbl_lim) tbl = __ldg(trow + warp + lane * kDecodeWarps);

    const int cap = min(prm.max_blocks_per_seq * kBlockSize, prm.max_context_len);
    const int c = clamp_context(c_raw, cap, p == 0 && hk == 0 && threadIdx.x == 0);
    const int parts = max(1, (c + prm.part_tokens - 1) / prm.part_tokens);
    if (p >= parts) return;

    const int nblk_seq = (c + kBlockSize - 1) / kBlockSize;
    const int nb_cta = max(0, min(nblk_seq - blk0, part_blocks));
    const int last_valid = c - (nblk_seq - 1) * kBlockSize;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *ring = smem + warp * C::WARP_RING;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bars = smem_addr(smem + C::OFF_BAR) + warp * C::NSTAGE * 8;
    float *pbuf = reinterpret_cast<float *>(smem + C::OFF_P + warp * C::PBUF);  // [16][G] of (p, p)
    const uint32_t pbuf_s = smem_addr(pbuf);

    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::NSTAGE; ++s) mbar_init(bars + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();

    // This warp's blocks: partition block warp + k * kDecodeWarps, k < nb_w.
    const int nb_w = nb_cta > warp ? (nb_cta - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
    uint32_t bad_mask = 0;

    auto issue = [&](int k) {
        if (k >= 32 && (k & 31) == 0) {
            const int li = warp + (k + lane) * kDecodeWarps;
            tbl = k + lane < nb_w && li < tbl_lim ? __ldg(trow + li) : 0;
        }
        int pb = __shfl_sync(0xffffffffu, tbl, k & 31);
        const int s = k % C::NSTAGE;
        if (pb < 0 || pb >= prm.num_blocks) {
            if (lane == 0) flag_status(PA_STATUS_BAD_BLOCK_ID);
            pb = 0;
            bad_mask |= 1u << s;
        } else {
            bad_mask &= ~(1u << s);
        }
        const uint32_t bar = bars + 8 * s;
        if (lane == 0) {
            mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
            const uint32_t dst = ring_s + s * C::STAGE_BYTES;
            tma_load_3d(dst, &tm_k, 0, hk, pb * kBlockSize, bar);
            tma_load_3d(dst + kBlockSize * C::R, &tm_v, 0, hk, pb * kBlockSize, bar);
        }
    };
    // L2 prefetch of block kp when it is inside the 32-entry table window of
    // block kw, the block issued last.
    auto prefetch = [&](int kp, int kw) {
        if (C::PF == 0 || kp >= nb_w || (kp >> 5) != (kw >> 5)) return;
        const int pb = __shfl_sync(0xffffffffu, tbl, kp & 31);
        if (lane == 0 && pb >= 0 && pb < prm.num_blocks) {
            tma_prefetch_l2_3d(&tm_k, 0, hk, pb * kBlockSize);
            tma_prefetch_l2_3d(&tm_v, 0, hk, pb * kBlockSize);
        }
    };

    int issued = 0;
    for (; issued < min(C::NSTAGE, nb_w); ++issued) issue(issued);
    if (C::PF > 0) {
#pragma unroll 1
        for (int kp = C::NSTAGE; kp < C::NSTAGE + C::PF; ++kp) prefetch(kp, 0);
    }

    // Queries of the group in this lane's head order, pre-scaled by
    // scale * log2(e), as packed pairs of the lane's columns.
    f32x2 q2[G][P2];
    {
        constexpr int QV = C::VE * static_cast<int>(sizeof(Tq)) / 16;  // 16-byte q loads per chunk
        constexpr int QP = Widen<Tq>::N / 2;                            // pairs per q load
        const Tq *qb = static_cast<const Tq *>(prm.q) + (static_cast<size_t>(b) * prm.num_heads + hk * G) * D;
        const f32x2 sc = pack2(prm.scale_log2, prm.scale_log2);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const Tq *qh = qb + (g ^ hmask) * D;
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) {
#pragma unroll
                for (int u = 0; u < QV; ++u) {
                    const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(qh + (ch * C::L + j) * C::VE) + u);
                    Widen<Tq>::apply2(raw, &q2[g][ch * VP + u * QP]);
                }
#pragma unroll
                for (int e = 0; e < VP; ++e) mul2(q2[g][ch * VP + e], sc);
            }
        }
    }

    f32x2 acc2[G][P2];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < P2; ++e) acc2[g][e] = 0ull;
    float m_col = -CUDART_INF_F;  // running max (log2 domain) of head lane % G
    float l_f[C::NFIN];           // this lane's share of the running sums of heads hmask + f
    float mu_f[C::NFIN];          // exponent reference of head hmask + f: its max, or 0 while -inf
    float thr_f[C::NFIN];         // a score above this moves the max of head hmask + f
#pragma unroll
    for (int f = 0; f < C::NFIN; ++f) {
        l_f[f] = 0.f;
        mu_f[f] = 0.f;
        thr_f[f] = -CUDART_INF_F;
    }
    const int t_own = smask * C::RS + rg;  // the row of this lane's scores
    const uint32_t p_own = pbuf_s + (t_own * G + hmask) * 8;

    int k = 0;
    bool failed = false;
    for (; k < nb_w; ++k) {
        const int s = k % C::NSTAGE;
        const bool landed = mbar_wait(bars + 8 * s, (k / C::NSTAGE) & 1);
        if (!__all_sync(0xffffffffu, landed)) {
            failed = true;
            break;
        }
        const int lblk = blk0 + warp + k * kDecodeWarps;
        const int n_valid = ((bad_mask >> s) & 1u) ? 0 : (lblk == nblk_seq - 1 ? last_valid : kBlockSize);
        unsigned char *kb = ring + s * C::STAGE_BYTES;
        unsigned char *vb = kb + kBlockSize * C::R;
        if (n_valid < kBlockSize) {
            if (n_valid == 0) {  // a table entry outside the pool: nothing of this block is used
                __syncwarp();
                if (issued < nb_w) issue(issued++);
                continue;
            }
            // Rows past the context may hold anything (NaN included) and have
            // probability 0: clear their V so that 0 * V adds nothing.
            for (int i = n_valid * (C::R / 16) + lane; i < kBlockSize * (C::R / 16); i += 32)
                reinterpret_cast<uint4 *>(vb)[i] = make_uint4(0u, 0u, 0u, 0u);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }

        // ---- scores: q . k for the G heads, this lane's columns, steps in lane
        // order. Step slots s and s + STEPS/2 meet at the first reduce step, so
        // they are computed together and reduced at once (fewer live partials).
        auto qk_step = [&](int st, float (&a)[G]) {
            const int row = (st ^ smask) * C::RS + rg;
            f32x2 s2[G];
#pragma unroll
            for (int g = 0; g < G; ++g) s2[g] = 0ull;
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) {
                f32x2 k2[VP];
                load_chunk<Tc, C::CB>(kb + row * C::R + (ch * C::L + j) * C::CB, k2);
#pragma unroll
                for (int e = 0; e < VP; ++e)
#pragma unroll
                    for (int g = 0; g < G; ++g) fma2(s2[g], q2[g][ch * VP + e], k2[e]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float a0, a1;
                unpack2(s2[g], a0, a1);
                a[g] = a0 + a1;
            }
        };
        float part[C::NPART / 2];
#pragma unroll
        for (int st = 0; st < C::STEPS / 2; ++st) {
            float lo[G], hi[G];
            qk_step(st, lo);
            qk_step(st + C::STEPS / 2, hi);
#pragma unroll
            for (int g = 0; g < G; ++g) part[st * G + g] = lo[g] + __shfl_xor_sync(0xffffffffu, hi[g], C::L / 2);
        }
        TransposeReduce<C::NPART / 2, C::L / 4>::run(part);
        float sc[C::NFIN];
#pragma unroll
        for (int f = 0; f < C::NFIN; ++f) sc[f] = part[f];
        if (n_valid < kBlockSize && t_own >= n_valid) {
#pragma unroll
            for (int f = 0; f < C::NFIN; ++f) sc[f] = -CUDART_INF_F;
        }

        // ---- online softmax. The max of a head moves (and O, l are rescaled)
        // only when one of its scores exceeds it by more than 8 (a factor 256
        // in probability); otherwise the older max is kept and P stays below
        // 2^8. The result is the same softmax, with fewer rescales.
        bool grow = false;
#pragma unroll
        for (int f = 0; f < C::NFIN; ++f) grow |= sc[f] > thr_f[f];
        if (__any_sync(0xffffffffu, grow)) {
            // Block maxima through the buffer: scores in, one head per lane column.
#pragma unroll
            for (int f = 0; f < C::NFIN; ++f) pbuf[(t_own * G + hmask + f) * 2] = sc[f];
            __syncwarp();
            constexpr int ENT = (kBlockSize * G + 31) / 32;
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int e = 0; e < ENT; ++e) {
                const int idx = lane + 32 * e;
                if (idx < kBlockSize * G) mx = fmaxf(mx, pbuf[idx * 2]);
            }
#pragma unroll
            for (int off = G; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_col, mx);
            const float alpha = m_new == -CUDART_INF_F ? 1.f : exp2f(m_col - m_new);
            m_col = m_new;
#pragma unroll
            for (int g = 0; g < G; ++g) {  // lane g holds head g's values
                const float a = __shfl_sync(0xffffffffu, alpha, g);
                const f32x2 a2 = pack2(a, a);
#pragma unroll
                for (int e = 0; e < P2; ++e) mul2(acc2[g][e], a2);
            }
#pragma unroll
            for (int f = 0; f < C::NFIN; ++f) {
                const float mf = __shfl_sync(0xffffffffu, m_col, hmask + f);
                l_f[f] *= __shfl_sync(0xffffffffu, alpha, hmask + f);
                mu_f[f] = mf == -CUDART_INF_F ? 0.f : mf;
                thr_f[f] = mf + 8.f;
            }
            __syncwarp();  // every lane has read the scores before they are overwritten
        }
        // probabilities, stored as (p, p) pairs for the packed P.V
        if constexpr (C::NFIN == 1) {
            const float p0 = ex2_approx(sc[0] - mu_f[0]);
            l_f[0] += p0;
            asm volatile("st.shared.v2.f32 [%0], {%1, %1};" ::"r"(p_own), "f"(p0) : "memory");
        } else {
#pragma unroll
            for (int f = 0; f < C::NFIN; f += 2) {
                const float p0 = ex2_approx(sc[f] - mu_f[f]);
                const float p1 = ex2_approx(sc[f + 1] - mu_f[f + 1]);
                l_f[f] += p0;
                l_f[f + 1] += p1;
                asm volatile("st.shared.v4.f32 [%0], {%1, %1, %2, %2};" ::"r"(p_own + f * 8), "f"(p0), "f"(p1)
                             : "memory");
            }
        }
        __syncwarp();

        // ---- O += P . V
#pragma unroll
        for (int st = 0; st < C::STEPS; ++st) {
            const int t = st * C::RS + rg;
            f32x2 pr[G];
            if constexpr (G == 1) {
                pr[0] = lds_pair(pbuf_s + t * 8);
            } else {
#pragma unroll
                for (int g = 0; g < G; g += 2) lds_pair2(pbuf_s + (t * G + g) * 8, pr[g], pr[g + 1]);
            }
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) {
                f32x2 v2[VP];
                load_chunk<Tc, C::CB>(vb + t * C::R + (ch * C::L + j) * C::CB, v2);
#pragma unroll
                for (int e = 0; e < VP; ++e)
#pragma unroll
                    for (int g = 0; g < G; ++g) fma2(acc2[g][ch * VP + e], pr[g], v2[e]);
            }
        }
        __syncwarp();
        if (issued < nb_w) {
            issue(issued);
            if (C::PF > 0) prefetch(issued + C::PF, issued);
            ++issued;
        }
    }
    if (failed) {
        // Let copies still in flight land before the ring is reused.
        for (int kk = k; kk < issued; ++kk) mbar_wait(bars + 8 * (kk % C::NSTAGE), (kk / C::NSTAGE) & 1);
    }

    // ---- merge the warps (and each warp's row groups) of this CTA
    if (C::DUP > 1 && (j & (C::DUP - 1)) != 0) {
#pragma unroll
        for (int f = 0; f < C::NFIN; ++f) l_f[f] = 0.f;  // a copy of another lane's sums
    }
    float l_head[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float x = 0.f;
#pragma unroll
        for (int f = 0; f < C::NFIN; ++f) x += (g == hmask + f) ? l_f[f] : 0.f;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        l_head[g] = x;
    }
    __syncthreads();
    float *red_acc = reinterpret_cast<float *>(smem);  // [warp][rg][g][D]
    float *red_m = reinterpret_cast<float *>(smem + C::OFF_ML);
    float *red_l = red_m + kDecodeWarps * G;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float mg = __shfl_sync(0xffffffffu, m_col, g);
        if (lane == 0) {
            red_m[warp * G + g] = mg;
            red_l[warp * G + g] = l_head[g];
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int ch = 0; ch < C::CH; ++ch) {
            float *dst = red_acc + ((warp * C::RS + rg) * G + g) * D + (ch * C::L + j) * C::VE;
#pragma unroll
            for (int e = 0; e < VP; e += 2) {
                float x0, x1, x2, x3;
                unpack2(acc2[g][ch * VP + e], x0, x1);
                unpack2(acc2[g][ch * VP + e + 1], x2, x3);
                *reinterpret_cast<float4 *>(dst + 2 * e) = make_float4(x0, x1, x2, x3);
            }
        }
    __syncthreads();

    for (int idx = threadIdx.x; idx < G * D; idx += kDecodeThreads) {
        const int g = idx / D, d = idx % D;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, red_m[w * G + g]);
        float O = 0.f, Lsum = 0.f;
        if (M != -CUDART_INF_F) {
#pragma unroll
            for (int w = 0; w < kDecodeWarps; ++w) {
                const float mw = red_m[w * G + g];
                if (mw == -CUDART_INF_F) continue;
                const float wt = exp2f(mw - M);
                float o = 0.f;
#pragma unroll
                for (int r = 0; r < C::RS; ++r) o += red_acc[((w * C::RS + r) * G + g) * D + d];
                O += wt * o;
                Lsum += wt * red_l[w * G + g];
            }
        }
        O *= prm.v_scale;
        const int h = hk * G + g;
        if (parts == 1) {
            Tq *out = static_cast<Tq *>(prm.out) + (static_cast<size_t>(b) * prm.num_heads + h) * D + d;
            store_out(out, Lsum > 0.f ? O / Lsum : 0.f);
        } else {
            const size_t pi = (static_cast<size_t>(b) * prm.num_heads + h) * prm.max_parts + p;
            prm.ws_o[pi * D + d] = O;
            if (d == 0) {
                prm.ws_m[pi] = M;
                prm.ws_l[pi] = Lsum;
            }
        }
    }
    if (parts == 1 || !prm.fuse_merge) return;

    // ---- fused merge: the last CTA of this (sequence, KV head) to finish merges
    // every partition's partials. Partials are published (fence) before the
    // ticket is taken, and read from L2 after it. A ticket is the call's stamp
    // and the arrivals so far; one with another stamp (an earlier call, or
    // memory never used as a ticket) counts as no arrivals, so the workspace
    // needs no initialisation.
    int *flag = reinterpret_cast<int *>(smem + C::OFF_FLAG);
    unsigned long long *ticket = prm.ws_ticket + static_cast<size_t>(b) * prm.num_kv_heads + hk;
    const unsigned long long stamp = static_cast<unsigned long long>(prm.stamp) << 32;
    __syncthreads();  // the CTA's partial writes happen before thread 0's fence (cumulativity)
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned long long cur = __ldcg(ticket), seen;
        unsigned int n;
        do {
            seen = cur;
            n = (seen & 0xffffffff00000000ull) == stamp ? static_cast<unsigned int>(seen) : 0u;
            cur = atomicCAS(ticket, seen, stamp | (n + 1u));
        } while (cur != seen);
        if (n >= static_cast<unsigned int>(parts)) flag_status(PA_STATUS_BAD_WORKSPACE);
        *flag = n + 1u == static_cast<unsigned int>(parts);
    }
    __syncthreads();
    if (!*flag) return;
    __threadfence();
    merge_partitions_n<Tq, (G * D + kDecodeThreads - 1) / kDecodeThreads>(prm, b, hk * G, threadIdx.x,
                                                                          kDecodeThreads, G * D, parts, D);
    if (threadIdx.x == 0) atomicExch(ticket, stamp);  // no arrivals: a replay of this call starts afresh
}

// Merge the partitions of every sequence that has more than one (the merge of
// pa_decode_merge, a kernel of its own). Grid (KV head, sequence), G * D
// threads: one per output element of the group. It is launched as a
// programmatic dependent of decode_kernel and waits for it
// (griddepcontrol.wait) before reading the partials.
template <typename T>
__global__ void decode_reduce_kernel(const DecodeParams prm, int D) {
    // context_lens was written before decode_kernel ran (decode_kernel waited for
    // it), so it may be read before waiting for decode_kernel's partials.
    const int hk = blockIdx.x, b = blockIdx.y;
    const int G = prm.num_heads / prm.num_kv_heads;
    const int g = threadIdx.x / D, d = threadIdx.x % D;
    const int cap = min(prm.max_blocks_per_seq * kBlockSize, prm.max_context_len);
    const int c = clamp_context(__ldg(prm.context_lens + b), cap, false);
    const int parts = max(1, (c + prm.part_tokens - 1) / prm.part_tokens);
    if (parts == 1 || g >= G) return;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    merge_partitions<T>(prm, b, hk * G + g, parts, d, D);
}

}  // namespace pa
