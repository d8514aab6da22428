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
//    Sequences longer than a partition also write (m, l, O) partials, and
//    decode_reduce_kernel merges them.
//  * Every query head of the KV head's group (G = H / Hk of them) reads each
//    loaded block from shared memory, so K/V cross HBM once per KV head.
//  * The 4 warps of a CTA take the partition's blocks round-robin. Each warp
//    streams its own blocks through an NSTAGE-deep shared-memory ring. A
//    block's 16 K rows and 16 V rows of one KV head are two TMA tiled loads
//    (a [16][D] box of the pool viewed as [NB*16][Hk][D]) into a ring slot,
//    and an mbarrier counts the bytes. Fetches run NSTAGE blocks ahead, so
//    the table entry, the HBM fetch and the math of different blocks overlap.
//  * Lanes own column slices of a row made of CH chunks of 16 bytes (8 for
//    FP8 rows with groups of 8 heads; CH = 2, or 1 for groups of 8 heads and
//    FP8 rows, to bound registers), interleaved so shared-memory
//    reads are conflict free. L = row_bytes / (16 * CH) lanes cover a row and RS = 32 / L rows are processed per step. q.k
//    partial sums are folded across the L lanes with a transpose-reduce
//    (each shuffle step halves the values per lane). Softmax runs in fp32
//    (exp2 with scale * log2(e) folded into q). P.V uses packed two-wide
//    fp32 FMAs.
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
    static constexpr int STAGE_BYTES = 2 * kBlockSize * R; // K and V of one block
    // Two stages per warp and three CTAs per SM (12 warps) measured faster on
    // B200 than three stages at two CTAs per SM: more warps hide the math's
    // latency better, and 12 x 2 x 8 KB in flight covers HBM latency.
    static constexpr int NSTAGE = 2;
    // CTAs per SM the register budget is sized for (wide rows keep more live state).
    static constexpr int MIN_BLOCKS = G <= 4 ? 3 : 2;
    static constexpr int WARP_RING = NSTAGE * STAGE_BYTES;
    static constexpr int RING_BYTES = kDecodeWarps * WARP_RING;
    static constexpr int NPART = STEPS * G;                // q.k partials per lane per block
    static constexpr int NFIN = NPART >= L ? NPART / L : 1; // fully reduced scores per lane
    static constexpr int ENT = (kBlockSize * G) / 32 > 0 ? (kBlockSize * G) / 32 : 1;
    static constexpr int RED_BYTES = kDecodeWarps * RS * G * D * 4;
    static constexpr int BIG = RING_BYTES > RED_BYTES ? RING_BYTES : RED_BYTES;
    static constexpr int OFF_BAR = BIG;
    static constexpr int OFF_S = OFF_BAR + kDecodeWarps * NSTAGE * 8;
    static constexpr int OFF_ML = OFF_S + kDecodeWarps * kBlockSize * G * 4;
    static constexpr int SMEM = OFF_ML + 2 * kDecodeWarps * G * 4;
    static_assert(R % (CB * CH) == 0 && L >= 1 && L <= 32 && 32 % L == 0, "row must split into lane slices");
    static_assert(kBlockSize % RS == 0, "rows per step must divide the block");
    static_assert(32 % G == 0 && G <= 8, "group size");
};

// Sum N values per lane across groups of lanes that differ in the bits of
// OFF, OFF/2, ..., 1. Every step sends half of the remaining values to the
// partner lane and keeps the other half, so the lane ends with
// max(1, N / (2*OFF)) fully summed values. `base` gets the index (into the
// original N) of the first one.
template <int N, int OFF>
struct TransposeReduce {
    template <int NA>
    __device__ __forceinline__ static void run(float (&v)[NA], int lane, int &base) {
        if constexpr (OFF == 0) {
            return;
        } else if constexpr (N > 1) {
            constexpr int H = N / 2;
            const bool upper = (lane & OFF) != 0;
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const float send = upper ? v[i] : v[i + H];
                const float keep = upper ? v[i + H] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
            }
            if (upper) base += H;
            TransposeReduce<H, OFF / 2>::run(v, lane, base);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
            TransposeReduce<1, OFF / 2>::run(v, lane, base);
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
    long long num_blocks;
    int max_blocks_per_seq;
    int num_heads;
    int num_kv_heads;
    int max_context_len;
    int part_tokens;
    int max_parts;
    float scale_log2;  // softmax scale * log2(e) (times k_scale for an FP8 cache)
    float v_scale;     // 1, or the FP8 value scale
};

// Tq: element type of q and out. Tc: element type of the caches (the same, or
// FP8 E4M3 codes with bf16 q/out).
template <typename Tq, typename Tc, int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, DecodeCfg<Tc, D, G>::MIN_BLOCKS)
    decode_kernel(const DecodeParams prm, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v) {
    using C = DecodeCfg<Tc, D, G>;
    // Grid (KV head, sequence, partition): every unit's first partition launches
    // before any second one, so full partitions run first and the short last
    // partitions (or empty CTAs) form the tail.
    const int hk = blockIdx.x, b = blockIdx.y, p = blockIdx.z;
    // Launched as a programmatic dependent (its launch overlaps the previous
    // kernel, e.g. the cache write): wait for that kernel before reading any input.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // The merge kernel may be scheduled as soon as every CTA of this grid has
    // started; it still waits for this grid to finish before reading partials.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int cap = min(prm.max_blocks_per_seq * kBlockSize, prm.max_context_len);
    const int c = clamp_context(__ldg(prm.context_lens + b), cap, p == 0 && hk == 0 && threadIdx.x == 0);
    const int parts = max(1, (c + prm.part_tokens - 1) / prm.part_tokens);
    if (p >= parts) return;

    const int part_blocks = prm.part_tokens / kBlockSize;
    const int nblk_seq = (c + kBlockSize - 1) / kBlockSize;
    const int blk0 = p * part_blocks;
    const int nb_cta = max(0, min(nblk_seq - blk0, part_blocks));
    const int last_valid = c - (nblk_seq - 1) * kBlockSize;

    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int rg = lane / C::L, j = lane % C::L;

    unsigned char *ring = smem + warp * C::WARP_RING;
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bars = smem_addr(smem + C::OFF_BAR) + warp * C::NSTAGE * 8;
    float *s_buf = reinterpret_cast<float *>(smem + C::OFF_S) + warp * kBlockSize * G;

    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::NSTAGE; ++s) mbar_init(bars + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();

    // This warp's blocks: partition block warp + k * kDecodeWarps, k < nb_w.
    const int nb_w = nb_cta > warp ? (nb_cta - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
    const int *trow = prm.block_tables + static_cast<size_t>(b) * prm.max_blocks_per_seq + blk0;
    int tbl = lane < nb_w ? __ldg(trow + warp + lane * kDecodeWarps) : 0;
    uint32_t bad_mask = 0;

    auto issue = [&](int k) {
        if (k >= 32 && (k & 31) == 0)
            tbl = k + lane < nb_w ? __ldg(trow + warp + (k + lane) * kDecodeWarps) : 0;
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

    // Queries of the group, pre-scaled by scale * log2(e), as packed pairs.
    constexpr int P2 = C::EPL / 2;  // packed pairs per lane per row
    constexpr int VP = C::VE / 2;   // packed pairs per chunk
    f32x2 q2[G][P2];
    {
        // the lane's dims in q: the same VE-element chunks as in the cache row
        constexpr int QV = C::VE * static_cast<int>(sizeof(Tq)) / 16;  // 16-byte q loads per chunk
        constexpr int QP = Widen<Tq>::N / 2;                            // pairs per q load
        const Tq *qb = static_cast<const Tq *>(prm.q) + (static_cast<size_t>(b) * prm.num_heads + hk * G) * D;
        const f32x2 sc = pack2(prm.scale_log2, prm.scale_log2);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) {
#pragma unroll
                for (int u = 0; u < QV; ++u) {
                    const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(qb + g * D + (ch * C::L + j) * C::VE) + u);
                    Widen<Tq>::apply2(raw, &q2[g][ch * VP + u * QP]);
                }
#pragma unroll
                for (int e = 0; e < VP; ++e) mul2(q2[g][ch * VP + e], sc);
            }
    }

    f32x2 acc2[G][P2];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < P2; ++e) acc2[g][e] = 0ull;
    float m_own = -CUDART_INF_F;  // running max of head lane % G (log2 domain)
    float l_own = 0.f;            // this lane's share of that head's running sum

    int issued = 0;
    for (; issued < min(C::NSTAGE, nb_w); ++issued) issue(issued);

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
        const unsigned char *kb = ring + s * C::STAGE_BYTES;
        const unsigned char *vb = kb + kBlockSize * C::R;

        // ---- scores: q . k for the G heads and this lane's rows
        float part[C::NPART];
#pragma unroll
        for (int st = 0; st < C::STEPS; ++st) {
            const int row = st * C::RS + rg;
            f32x2 k2[P2];
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) load_chunk<Tc, C::CB>(kb + row * C::R + (ch * C::L + j) * C::CB, &k2[ch * VP]);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                f32x2 s2 = 0ull;
#pragma unroll
                for (int e = 0; e < P2; ++e) fma2(s2, q2[g][e], k2[e]);
                float a0, a1;
                unpack2(s2, a0, a1);
                part[st * G + g] = a0 + a1;
            }
        }
        int base = 0;
        TransposeReduce<C::NPART, C::L / 2>::run(part, lane, base);
#pragma unroll
        for (int f = 0; f < C::NFIN; ++f) {
            const int idx = base + f;
            const int t = (idx / G) * C::RS + rg;
            s_buf[t * G + idx % G] = t < n_valid ? part[f] : -CUDART_INF_F;
        }
        __syncwarp();

        // ---- online softmax for head lane % G over this block. The reference max
        // m_own is updated (and O, l rescaled) only when a score exceeds it by more
        // than 8 in the exp2 domain; otherwise the older max is kept and P stays
        // below 2^8. The result is the same softmax, with fewer rescales.
        float sv[C::ENT];
        bool grow = false;
#pragma unroll
        for (int e = 0; e < C::ENT; ++e) {
            const int idx = lane + 32 * e;
            sv[e] = idx < kBlockSize * G ? s_buf[idx] : -CUDART_INF_F;
            grow |= sv[e] > m_own + 8.f;
        }
        if (__any_sync(0xffffffffu, grow)) {
            float mx = -CUDART_INF_F;
#pragma unroll
            for (int e = 0; e < C::ENT; ++e) mx = fmaxf(mx, sv[e]);
#pragma unroll
            for (int off = G; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_own, mx);
            const float alpha = m_own == -CUDART_INF_F ? 0.f : exp2f(m_own - m_new);
            l_own *= alpha;
            m_own = m_new;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float a = __shfl_sync(0xffffffffu, alpha, g);
                const f32x2 a2 = pack2(a, a);
#pragma unroll
                for (int e = 0; e < P2; ++e) mul2(acc2[g][e], a2);
            }
        }
        float psum = 0.f;
        if (m_own != -CUDART_INF_F) {
#pragma unroll
            for (int e = 0; e < C::ENT; ++e) {
                sv[e] = exp2f(sv[e] - m_own);
                psum += sv[e];
            }
        } else {
#pragma unroll
            for (int e = 0; e < C::ENT; ++e) sv[e] = 0.f;
        }
        l_own += psum;
#pragma unroll
        for (int e = 0; e < C::ENT; ++e) {
            const int idx = lane + 32 * e;
            if (idx < kBlockSize * G) s_buf[idx] = sv[e];
        }
        __syncwarp();

        // ---- O += P . V
#pragma unroll
        for (int st = 0; st < C::STEPS; ++st) {
            const int t = st * C::RS + rg;
            float pr[G];
#pragma unroll
            for (int g = 0; g < G; ++g) pr[g] = s_buf[t * G + g];
            f32x2 v2[P2];
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) load_chunk<Tc, C::CB>(vb + t * C::R + (ch * C::L + j) * C::CB, &v2[ch * VP]);
            if (t < n_valid) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const f32x2 p2 = pack2(pr[g], pr[g]);
#pragma unroll
                    for (int e = 0; e < P2; ++e) fma2(acc2[g][e], p2, v2[e]);
                }
            }
        }
        __syncwarp();
        if (issued < nb_w) issue(issued++);
    }
    if (failed) {
        // Let copies still in flight land before the ring is reused.
        for (int kk = k; kk < issued; ++kk) mbar_wait(bars + 8 * (kk % C::NSTAGE), (kk / C::NSTAGE) & 1);
    }

    // ---- merge the warps (and each warp's row groups) of this CTA
#pragma unroll
    for (int off = G; off < 32; off <<= 1) l_own += __shfl_xor_sync(0xffffffffu, l_own, off);
    __syncthreads();
    float *red_acc = reinterpret_cast<float *>(smem);  // [warp][rg][g][D]
    float *red_m = reinterpret_cast<float *>(smem + C::OFF_ML);
    float *red_l = red_m + kDecodeWarps * G;
    if (lane < G) {
        red_m[warp * G + lane] = m_own;
        red_l[warp * G + lane] = l_own;
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
}

// Merge the partitions of every sequence that has more than one:
//   M = max_p m_p,  L = sum_p 2^(m_p - M) l_p,  out = sum_p 2^(m_p - M) O_p / L.
// Grid (KV head, sequence), G * D threads: one per output element of the group.
// It is launched as a programmatic dependent of decode_kernel and waits for it
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
    const int h = hk * G + g;
    const size_t base = (static_cast<size_t>(b) * prm.num_heads + h) * prm.max_parts;
    // one pass with a running max: the loads of up to 8 partitions go out together
    float M = -CUDART_INF_F, O = 0.f, L = 0.f;
    for (int p0 = 0; p0 < parts; p0 += 8) {
        float mp[8], lp[8], op[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool in = p0 + i < parts;
            mp[i] = in ? prm.ws_m[base + p0 + i] : -CUDART_INF_F;
            lp[i] = in ? prm.ws_l[base + p0 + i] : 0.f;
            op[i] = in ? prm.ws_o[(base + p0 + i) * D + d] : 0.f;
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

}  // namespace pa
