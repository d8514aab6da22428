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
// How it runs on B200 (two kernels, the second a programmatic dependent):
//  * Work is the flat list of (sequence, KV head, block) triples in that
//    order; a (sequence, KV head) pair is a "unit". The grid is persistent:
//    one CTA of WARPS warps per SM (12 for groups of up to 4 heads), and
//    each warp takes one of WARPS * gridDim.x equal, contiguous slices of
//    the list, so every warp gets the same number of blocks (to one)
//    whatever the mix of lengths: no tail of short CTAs, no empty CTAs, one
//    prologue per CTA. A CTA finds its warps' slices by a prefix sum of the
//    sequences' block counts, read from context_lens on the device, and one
//    binary search per warp. After that the warps run independently.
//  * A unit's part inside one slice is a "segment". A warp leaving a segment
//    writes the unit's output itself when the whole unit lies in its slice;
//    otherwise it writes the segment's partial (m, l, O) to the workspace.
//    decode_merge_kernel then merges the partials of every cut unit.
//  * Every query head of the KV head's group (G = H / Hk of them) reads each
//    loaded block from shared memory, so K/V cross HBM once per KV head.
//  * Each warp streams its blocks through an NSTAGE-deep shared-memory ring:
//    a block's 16 K rows and 16 V rows of one KV head are two TMA tiled loads
//    (a [16][D] box of the pool viewed as [NB*16][Hk][D]) into a ring slot,
//    and an mbarrier counts the bytes. Fetches run NSTAGE blocks ahead,
//    across segment boundaries. The first block of a segment also brings the
//    unit's G query rows (a bulk copy into the stage's query slot).
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
#pragma once

#include <math_constants.h>

#include "pa_common.cuh"
#include "tmap.cuh"

namespace pa {

// Dynamic shared memory one CTA may use on sm_100.
constexpr int kCtaSmem = 227 * 1024;

template <typename T, int D, int G>
struct DecodeCfg {
    static constexpr int E = sizeof(T);
    static constexpr int R = D * E;                        // bytes of one token row of one KV head
    // Bytes of one chunk: 16, or 8 for FP8 rows, so that a lane holds 8 dims
    // per chunk as for bf16 (16 would spill q and O).
    static constexpr int CB = E == 1 ? 8 : 16;
    // One chunk per lane and row: q and O then take 64 registers for 4 heads
    // (two chunks spill at 12 warps per SM).
    static constexpr int CH = 1;
    static constexpr int L = R / (CB * CH);                // lanes covering one row
    static constexpr int RS = 32 / L;                      // rows per warp step
    static constexpr int STEPS = kBlockSize / RS;          // steps per block
    static constexpr int VE = CB / E;                      // elements per chunk
    static constexpr int EPL = CH * VE;                    // elements per lane per row
    static constexpr int P2 = EPL / 2;                     // packed pairs per lane per row
    static constexpr int STAGE_BYTES = 2 * kBlockSize * R; // K and V of one block
    // Two stages per warp at 12 warps per SM measured faster on B200 than
    // three stages at 8 warps or four at 6 (the same bytes in flight).
    static constexpr int NSTAGE = 2;
    static constexpr int WARP_RING = NSTAGE * STAGE_BYTES;
    static constexpr int NPART = STEPS * G;                 // q.k partials per lane per block
    static constexpr int NFIN = NPART >= L ? NPART / L : 1; // complete scores per lane
    static constexpr int DUP = NPART >= L ? 1 : L / NPART;  // lanes holding the same scores
    static constexpr int PBUF = kBlockSize * G * 8;         // per warp: [16 rows][G heads] of (p, p)
    // One unit's queries (bf16 with an FP8 cache), fetched with the first block
    // of each segment into that block's stage.
    static constexpr int QBYTES = G * D * (E == 1 ? 2 : E);
    static constexpr int WARP_Q = NSTAGE * QBYTES;
    // Warps of one CTA, the CTA filling its SM: 12 (8 for wide groups, whose
    // live state takes more registers), or fewer where their rings would not
    // fit in shared memory (fp32 rows of 128). One CTA of 12 warps measured
    // faster on B200 than three CTAs of 4 with the same rings.
    static constexpr int WARPS_REG = G <= 4 ? 12 : 8;
    static constexpr int WARPS_SMEM = (kCtaSmem - 1024) / (WARP_RING + WARP_Q + PBUF + NSTAGE * 8 + 20);
    static constexpr int WARPS = WARPS_REG < WARPS_SMEM ? WARPS_REG : WARPS_SMEM;
    static constexpr int THREADS = 32 * WARPS;
    static constexpr int RING_BYTES = WARPS * WARP_RING;
    static constexpr int OFF_Q = RING_BYTES;                // NSTAGE query slots per warp
    static constexpr int OFF_BAR = OFF_Q + WARPS * WARP_Q;  // NSTAGE mbarriers per warp
    static constexpr int OFF_P = OFF_BAR + (WARPS * NSTAGE * 8 + 15) / 16 * 16;
    static constexpr int OFF_MISC = OFF_P + WARPS * PBUF;   // the warps' slice starts
    static constexpr int SMEM = OFF_MISC + WARPS * 5 * 4 + 16;
    // CTAs of this kernel one SM holds, without a device to ask.
    static constexpr int RESIDENT = 1;
    static_assert(R % (CB * CH) == 0 && L >= 1 && L <= 32 && 32 % L == 0, "row must split into lane slices");
    static_assert(kBlockSize % RS == 0, "rows per step must divide the block");
    static_assert(32 % G == 0 && G <= 8, "group size");
    static_assert(G % NFIN == 0, "a lane's scores are consecutive heads of one row");
    static_assert(OFF_P % 16 == 0 && OFF_MISC % 16 == 0 && QBYTES % 16 == 0, "shared-memory alignment");
    static_assert(STEPS >= 2 && L >= 4, "the first reduce step pairs step slots s and s + STEPS / 2");
    static_assert(SMEM <= kCtaSmem && WARPS >= 1, "one CTA must fit an SM");
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

// A 16-byte store whose line L2 keeps over others (evict-last): for the partials
// the merge reads back while the K/V stream passes through L2 (measured on B200:
// the decode batch's call 63.6 -> 62.8 us).
__device__ __forceinline__ void st_v4_keep(float *p, float4 v) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w), "l"(pol)
                 : "memory");
}

struct DecodeParams {
    void *out;
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int *block_tables;
    const int *context_lens;
    float *ws_o;   // [slots][G][D] partial outputs; slot = slice index + unit index
    float *ws_m;   // [slots][G]
    float *ws_l;   // [slots][G]
    int *ws_unit;  // [B][Hk][2]: (first slice, slices) of each unit with blocks, written every call
    int warps_total;  // the decode kernel's warps (gridDim.x * WARPS): slices = min(warps_total, blocks)
    long long num_blocks;
    int num_seqs;
    int max_blocks_per_seq;
    int num_heads;
    int num_kv_heads;
    int max_context_len;
    float scale_log2;  // softmax scale * log2(e) (times k_scale for an FP8 cache)
    float v_scale;     // 1, or the FP8 value scale
};

// Position in the flat (sequence, KV head, block) list.
struct Cursor {
    int r;      // flat index minus the slice's first index
    int b, hk;  // the unit
    int c;      // context length of b (clamped)
    int nblk;   // blocks of the unit
    int blk;    // block within the unit
};

__device__ __forceinline__ int decode_cap(const DecodeParams &prm) {
    return min(prm.max_blocks_per_seq * kBlockSize, prm.max_context_len);
}

// Move x forward by n positions; returns the number of units left behind.
// Sequences of length 0 hold no blocks and are stepped over.
__device__ __forceinline__ int cursor_advance(Cursor &x, int n, const DecodeParams &prm) {
    x.r += n;
    x.blk += n;
    int passed = 0;
    while (x.blk >= x.nblk) {
        x.blk -= x.nblk;
        ++passed;
        if (++x.hk == prm.num_kv_heads) {
            x.hk = 0;
            do {
                if (++x.b >= prm.num_seqs) {  // past the end of the list: never used for a block
                    x.nblk = 1 << 30;
                    return passed;
                }
                x.c = clamp_context(__ldg(prm.context_lens + x.b), decode_cap(prm), false);
            } while (x.c == 0);
            x.nblk = (x.c + kBlockSize - 1) / kBlockSize;
        }
    }
    return passed;
}

// Slice holding flat index f when N items are cut into W slices
// [s * N / W, (s + 1) * N / W).
__device__ __forceinline__ int slice_of(long long f, long long N, int W) {
    return static_cast<int>(((f + 1) * W - 1) / N);
}

// Tq: element type of q and out. Tc: element type of the caches (the same, or
// FP8 E4M3 codes with bf16 q/out).
template <typename Tq, typename Tc, int D, int G>
__global__ void __launch_bounds__(DecodeCfg<Tc, D, G>::THREADS, 1)
    decode_kernel(const DecodeParams prm, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v) {
    using C = DecodeCfg<Tc, D, G>;
    constexpr int P2 = C::P2;      // packed pairs per lane per row
    constexpr int VP = C::VE / 2;  // packed pairs per chunk
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int rg = lane / C::L, j = lane % C::L;
    const int B = prm.num_seqs, Hk = prm.num_kv_heads;
    const int cap = decode_cap(prm);

    extern __shared__ __align__(128) unsigned char smem[];
    int *starts = reinterpret_cast<int *>(smem + C::OFF_MISC);  // per warp: b, hk, blk, c, nblk of its first block

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
    // kernel, e.g. the cache write): wait for that kernel before reading any
    // input. The merge kernel that follows may start its launch at once; it
    // waits for this grid to finish before reading anything.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // While the prologue scans the lengths, bring the block tables towards L2
    // (each CTA a 1/gridDim share, 128-byte lines), so that a warp's first
    // table read after the prologue does not wait on HBM. Up to 8 MB of table.
    {
        const long long lines = (static_cast<long long>(prm.num_seqs) * prm.max_blocks_per_seq * 4 + 127) / 128;
        if (lines <= (8LL << 20) / 128) {
            const char *tb = reinterpret_cast<const char *>(prm.block_tables);
            for (long long i = blockIdx.x + static_cast<long long>(gridDim.x) * threadIdx.x; i < lines;
                 i += static_cast<long long>(gridDim.x) * C::THREADS)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(tb + i * 128));
        }
    }

    // ---- prologue (the whole CTA): the total block count N, the slices, and
    // the unit holding each warp's first block, from prefix sums of Hk * blocks
    // over the sequences, a chunk of sequences at a time in shared memory (the
    // ring is not in use yet). With more sequences than one chunk holds, a
    // first pass sums N.
    constexpr int CHUNK = C::RING_BYTES / 8;
    long long *cum = reinterpret_cast<long long *>(smem);
    long long N = 0;
    if (B > CHUNK) {
        long long part = 0;
        for (int b = threadIdx.x; b < B; b += C::THREADS) {
            const int c = clamp_context(__ldg(prm.context_lens + b), cap, false);
            part += (c + kBlockSize - 1) / kBlockSize;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (lane == 0) cum[warp] = part;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < C::WARPS; ++w) N += cum[w];
        N *= Hk;
        __syncthreads();
    }
    const int cta0 = static_cast<int>(blockIdx.x) * C::WARPS;  // first slice of this CTA
    int WS = 0;  // slices: at most one per block, so that none is empty (a unit's slices are then
                 // exactly those from the slice of its first block to that of its last)
    {
        long long base = 0;
        for (int c0 = 0; c0 < B; c0 += CHUNK) {
            const int n = min(CHUNK, B - c0);
            for (int i = threadIdx.x; i < n; i += C::THREADS) {
                const int c = clamp_context(__ldg(prm.context_lens + c0 + i), cap, blockIdx.x == 0);
                cum[i] = static_cast<long long>((c + kBlockSize - 1) / kBlockSize) * Hk;
            }
            __syncthreads();
            if (warp == 0) {  // inclusive scan, 32 entries per step
                long long carry = base;
                for (int i0 = 0; i0 < n; i0 += 32) {
                    long long v = i0 + lane < n ? cum[i0 + lane] : 0;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const long long t = __shfl_up_sync(0xffffffffu, v, off);
                        if (lane >= off) v += t;
                    }
                    v += carry;
                    if (i0 + lane < n) cum[i0 + lane] = v;
                    carry = __shfl_sync(0xffffffffu, v, 31);
                }
            }
            __syncthreads();
            if (B <= CHUNK) N = cum[n - 1];  // one chunk: the total comes with the scan
            WS = static_cast<int>(min(static_cast<long long>(gridDim.x) * C::WARPS, N));
            // a sequence of length 0 has no blocks: CTA b % gridDim.x writes its zero rows
            for (int i = threadIdx.x; i < n; i += C::THREADS) {
                const long long hi = cum[i], lo = i ? cum[i - 1] : base;
                const int b = c0 + i;
                if (lo >= hi && b % static_cast<int>(gridDim.x) == static_cast<int>(blockIdx.x)) {
                    Tq *o = static_cast<Tq *>(prm.out) + static_cast<size_t>(b) * prm.num_heads * D;
                    for (int e = 0; e < prm.num_heads * D; ++e) store_out(o + e, 0.f);
                }
            }
            // thread w: the first block of slice cta0 + w, if it lies in this chunk
            const int w = threadIdx.x;
            if (w < C::WARPS && cta0 + w < WS) {
                const long long f = N * (cta0 + w) / WS;
                if (f >= base && f < cum[n - 1]) {
                    int lo_i = 0, hi_i = n - 1;  // the first sequence whose inclusive sum exceeds f
                    while (lo_i < hi_i) {
                        const int mid = (lo_i + hi_i) / 2;
                        if (cum[mid] > f) hi_i = mid;
                        else lo_i = mid + 1;
                    }
                    const long long lo = lo_i ? cum[lo_i - 1] : base;
                    const int nblk = static_cast<int>((cum[lo_i] - lo) / Hk);
                    const long long r = f - lo;
                    starts[5 * w + 0] = c0 + lo_i;
                    starts[5 * w + 1] = static_cast<int>(r / nblk);
                    starts[5 * w + 2] = static_cast<int>(r % nblk);
                    starts[5 * w + 3] = clamp_context(__ldg(prm.context_lens + c0 + lo_i), cap, false);
                    starts[5 * w + 4] = nblk;
                }
            }
            base = cum[n - 1];
            __syncthreads();
        }
    }
    if (cta0 >= WS) return;
    // ---- from here on every warp runs alone on its slice
    const int slice = cta0 + warp;
    if (slice >= WS) return;
    const long long s_lo = N * slice / WS, s_hi = N * (slice + 1) / WS;
    const int nb_w = static_cast<int>(s_hi - s_lo);

    unsigned char *ring = smem + warp * C::WARP_RING;
    const uint32_t ring_s = smem_addr(ring);
    const unsigned char *qslots = smem + C::OFF_Q + warp * C::WARP_Q;
    const uint32_t q_s = smem_addr(qslots);
    const uint32_t bars = smem_addr(smem + C::OFF_BAR) + warp * C::NSTAGE * 8;
    float *pbuf = reinterpret_cast<float *>(smem + C::OFF_P + warp * C::PBUF);  // [16][G] of (p, p)
    const uint32_t pbuf_s = smem_addr(pbuf);
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::NSTAGE; ++s) mbar_init(bars + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    Cursor cc{0, starts[5 * warp], starts[5 * warp + 1], starts[5 * warp + 3], starts[5 * warp + 4],
              starts[5 * warp + 2]};

    // ---- issue side: block k of this warp at cursor ic (NSTAGE blocks ahead of
    // the block being consumed), with the next 32 table entries of its unit
    // (lane i holds block tbase + i)
    int tb_u = -1, tbase = 0, tw = 0;
    uint32_t bad_mask = 0;
    auto issue = [&](int k, const Cursor &ic, bool new_seg) {
        const int u = ic.b * Hk + ic.hk;
        if (u != tb_u || ic.blk >= tbase + 32) {
            tb_u = u;
            tbase = ic.blk;
            const int e = tbase + lane;
            tw = e < min(ic.nblk, prm.max_blocks_per_seq)
                     ? __ldg(prm.block_tables + static_cast<size_t>(ic.b) * prm.max_blocks_per_seq + e)
                     : 0;
        }
        int pb = __shfl_sync(0xffffffffu, tw, ic.blk - tbase);
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
            // the first block of a segment brings the unit's queries along
            mbar_arrive_expect_tx(bar, C::STAGE_BYTES + (new_seg ? C::QBYTES : 0));
            if (new_seg)
                bulk_g2s(q_s + s * C::QBYTES,
                         static_cast<const Tq *>(prm.q) + (static_cast<size_t>(ic.b) * prm.num_heads + ic.hk * G) * D,
                         C::QBYTES, bar);
            const uint32_t dst = ring_s + s * C::STAGE_BYTES;
            // with an explicit evict-normal L2 policy: on B200 these loads measured 1.5 to
            // 2.5 % faster across the decode workloads than the same loads without one
            const uint64_t pol = policy_evict_normal();
            tma_load_3d_policy(dst, &tm_k, 0, ic.hk, pb * kBlockSize, bar, pol);
            tma_load_3d_policy(dst + kBlockSize * C::R, &tm_v, 0, ic.hk, pb * kBlockSize, bar, pol);
        }
    };
    // the fetch side's cursor: the last block fetched, NSTAGE - 1 ahead of the consumer
    Cursor icur = cc;
    for (int i = 0; i < min(C::NSTAGE, nb_w); ++i) {
        const bool new_seg = i == 0 || cursor_advance(icur, 1, prm) > 0;
        issue(i, icur, new_seg);
    }

    // Queries of a unit in this lane's head order, pre-scaled by
    // scale * log2(e), as packed pairs of the lane's columns, from the query
    // slot of stage s.
    f32x2 q2[G][P2];
    auto load_q = [&](int s) {
        constexpr int QV = C::VE * static_cast<int>(sizeof(Tq)) / 16;  // 16-byte q loads per chunk
        constexpr int QP = Widen<Tq>::N / 2;                            // pairs per q load
        const Tq *qb = reinterpret_cast<const Tq *>(qslots + s * C::QBYTES);
        const f32x2 sc = pack2(prm.scale_log2, prm.scale_log2);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const Tq *qh = qb + (g ^ hmask) * D;
#pragma unroll
            for (int ch = 0; ch < C::CH; ++ch) {
#pragma unroll
                for (int u = 0; u < QV; ++u) {
                    const uint4 raw = *(reinterpret_cast<const uint4 *>(qh + (ch * C::L + j) * C::VE) + u);
                    Widen<Tq>::apply2(raw, &q2[g][ch * VP + u * QP]);
                }
#pragma unroll
                for (int e = 0; e < VP; ++e) mul2(q2[g][ch * VP + e], sc);
            }
        }
    };

    f32x2 acc2[G][P2];
    float m_col;           // running max (log2 domain) of head lane % G
    float l_f[C::NFIN];    // this lane's share of the running sums of heads hmask + f
    float mu_f[C::NFIN];   // exponent reference of head hmask + f: its max, or 0 while -inf
    float thr_f[C::NFIN];  // a score above this moves the max of head hmask + f
    auto reset_state = [&]() {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < P2; ++e) acc2[g][e] = 0ull;
        m_col = -CUDART_INF_F;
#pragma unroll
        for (int f = 0; f < C::NFIN; ++f) {
            l_f[f] = 0.f;
            mu_f[f] = 0.f;
            thr_f[f] = -CUDART_INF_F;
        }
    };
    const int t_own = smask * C::RS + rg;  // the row of this lane's scores
    const uint32_t p_own = pbuf_s + (t_own * G + hmask) * 8;

    // ---- leave the segment of the unit at cc: the unit's output if the whole
    // unit lies in this slice, else the segment's partial (m, l, O)
    auto close_segment = [&]() {
        // sum O over the row groups of the warp (lanes that differ in the row-group bits)
#pragma unroll
        for (int off = C::L; off < 32; off <<= 1)
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < P2; ++e) {
                    float lo, hi;
                    unpack2(acc2[g][e], lo, hi);
                    lo += __shfl_xor_sync(0xffffffffu, lo, off);
                    hi += __shfl_xor_sync(0xffffffffu, hi, off);
                    acc2[g][e] = pack2(lo, hi);
                }
        if (C::DUP > 1 && (j & (C::DUP - 1)) != 0) {
#pragma unroll
            for (int f = 0; f < C::NFIN; ++f) l_f[f] = 0.f;  // a copy of another lane's sums
        }
        float l_head[G], m_head[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float x = 0.f;
#pragma unroll
            for (int f = 0; f < C::NFIN; ++f) x += (g == hmask + f) ? l_f[f] : 0.f;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            l_head[g] = x;
            m_head[g] = __shfl_sync(0xffffffffu, m_col, g);
        }
        const long long u_lo = s_lo + cc.r - cc.blk, u_hi = u_lo + cc.nblk;  // the unit's positions
        const bool whole = u_lo >= s_lo && u_hi <= s_hi;
        const int u = cc.b * Hk + cc.hk;
        const size_t slot = static_cast<size_t>(slice) + u;
        if (rg == 0) {  // lanes of row group 0 hold the warp's O for their columns
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int d0 = j * C::VE;
                const float sc = whole ? (l_head[g] > 0.f ? prm.v_scale / l_head[g] : 0.f) : prm.v_scale;
#pragma unroll
                for (int e = 0; e < VP; e += 2) {
                    float x0, x1, x2, x3;
                    unpack2(acc2[g][e], x0, x1);
                    unpack2(acc2[g][e + 1], x2, x3);
                    const float4 o = make_float4(x0 * sc, x1 * sc, x2 * sc, x3 * sc);
                    if (whole) {
                        store_out4(static_cast<Tq *>(prm.out) +
                                       (static_cast<size_t>(cc.b) * prm.num_heads + cc.hk * G + g) * D + d0 + 2 * e,
                                   o);
                    } else {
                        st_v4_keep(prm.ws_o + (slot * G + g) * D + d0 + 2 * e, o);
                    }
                }
            }
        }
        if (!whole && lane < G) {
            float m = m_head[0], l = l_head[0];
#pragma unroll
            for (int g = 1; g < G; ++g)
                if (lane == g) {
                    m = m_head[g];
                    l = l_head[g];
                }
            prm.ws_m[slot * G + lane] = m;
            prm.ws_l[slot * G + lane] = l;
        }
        if (lane == 0 && u_lo >= s_lo) {  // the unit starts in this slice: where its partials are
            int *rec = prm.ws_unit + 2 * static_cast<size_t>(u);
            rec[0] = slice;
            rec[1] = whole ? 1 : slice_of(u_hi - 1, N, WS) - slice + 1;
        }
    };

    reset_state();
    bool need_q = true;
    int k = 0;
    for (; k < nb_w; ++k) {
        const int s = k % C::NSTAGE;
        const bool landed = mbar_wait(bars + 8 * s, (k / C::NSTAGE) & 1);
        if (!__all_sync(0xffffffffu, landed)) break;
        if (need_q) {  // the segment's first block: its queries came with it
            load_q(s);
            need_q = false;
        }
        const int last_valid = cc.c - (cc.nblk - 1) * kBlockSize;
        const int n_valid = ((bad_mask >> s) & 1u) ? 0 : (cc.blk == cc.nblk - 1 ? last_valid : kBlockSize);
        unsigned char *kb = ring + s * C::STAGE_BYTES;
        unsigned char *vb = kb + kBlockSize * C::R;
        if (n_valid > 0) {
            if (n_valid < kBlockSize) {
                // Rows past the context may hold anything (NaN included) and have
                // probability 0: clear their V so that 0 * V adds nothing.
                for (int i = n_valid * (C::R / 16) + lane; i < kBlockSize * (C::R / 16); i += 32)
                    reinterpret_cast<uint4 *>(vb)[i] = make_uint4(0u, 0u, 0u, 0u);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }

            // ---- scores: q . k for the G heads, this lane's columns, steps in lane
            // order. Step slots s and s + STEPS/2 meet at the first reduce step, so
            // they are computed together and reduced at once (fewer live partials).
            auto qk_step = [&](int st, float(&a)[G]) {
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
                    asm volatile("st.shared.v4.f32 [%0], {%1, %1, %2, %2};" ::"r"(p_own + f * 8), "f"(p0),
                                 "f"(p1)
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
        }
        __syncwarp();
        Cursor nx = cc;  // this warp's next block
        const int passed = k + 1 < nb_w ? cursor_advance(nx, 1, prm) : 0;
        if (k + C::NSTAGE < nb_w) {
            const bool new_seg = cursor_advance(icur, 1, prm) > 0;  // block k + NSTAGE starts a unit
            issue(k + C::NSTAGE, icur, new_seg);
        }
        // ---- the last block, or the next one in another unit: the segment closes
        if (passed > 0 || k + 1 == nb_w) {
            close_segment();
            reset_state();
            need_q = true;
        }
        cc = nx;
    }
    if (k < nb_w) {
        // A bounded wait gave up (the status word says why): let copies still in
        // flight land before the CTA ends.
        for (int kk = k; kk < min(k + C::NSTAGE, nb_w); ++kk)
            mbar_wait(bars + 8 * (kk % C::NSTAGE), (kk / C::NSTAGE) & 1);
    }
}

// Merge the partials of every unit cut by slice boundaries:
//   M = max_s m_s,  L = sum_s 2^(m_s - M) l_s,  out = sum_s 2^(m_s - M) O_s / L
// over the unit's slices s (slots first + u .. first + slices - 1 + u). Grid
// (units, G*D/128 column groups) of MG warps: a lane takes four consecutive
// columns of one head, warp w the slices w, w + MG, ... with every slot's
// loads of a round in flight together (up to 8 slots a round); with MG > 1,
// warp 0 combines the warps' results through shared memory (for units cut
// into many slices, as in long contexts). A programmatic dependent of
// decode_kernel: it waits for it before reading the workspace.
// Batches of at most this many sequences let each merge CTA find its unit's
// slices from the lengths before the wait; larger ones read the records.
constexpr int kMergeScanSeqs = 256;

template <typename T, int G, int D, int MG>
__global__ void __launch_bounds__(32 * MG) decode_merge_kernel(const DecodeParams prm) {
    __shared__ float4 sh_o[MG][32];
    __shared__ float sh_m[MG][32], sh_l[MG][32];
    const int u = blockIdx.x;
    const int b = u / prm.num_kv_heads, hk = u % prm.num_kv_heads;
    const int lane = threadIdx.x % 32, grp = threadIdx.x / 32;
    const int idx = 4 * (blockIdx.y * 32 + lane);
    const bool col = idx < G * D;  // the same for every warp: lanes past G * D only take part in the barrier
    const int cap = decode_cap(prm);
    const int c_b = clamp_context(__ldg(prm.context_lens + b), cap, false);
    if (c_b == 0) return;  // zero rows, written by the decode kernel
    int first, nseg;
    if (prm.num_seqs <= kMergeScanSeqs) {
        // The unit's slices from the lengths alone (inputs, not written by the
        // decode kernel), before the wait: the same sums as the decode kernel's
        // prologue. A unit in one slice needs no merge and leaves at once.
        long long below = 0, total = 0;
        for (int i = lane; i < prm.num_seqs; i += 32) {
            const int c = clamp_context(__ldg(prm.context_lens + i), cap, false);
            const long long n = static_cast<long long>((c + kBlockSize - 1) / kBlockSize) * prm.num_kv_heads;
            total += n;
            below += i < b ? n : 0;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            total += __shfl_xor_sync(0xffffffffu, total, off);
            below += __shfl_xor_sync(0xffffffffu, below, off);
        }
        const int nblk = (c_b + kBlockSize - 1) / kBlockSize;
        const long long u_lo = below + static_cast<long long>(hk) * nblk;
        const int ws = static_cast<int>(min(static_cast<long long>(prm.warps_total), total));
        first = slice_of(u_lo, total, ws);
        nseg = slice_of(u_lo + nblk - 1, total, ws) - first + 1;
        if (nseg <= 1) return;  // a whole unit: written by the decode kernel
        asm volatile("griddepcontrol.wait;" ::: "memory");
    } else {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        first = __ldcg(prm.ws_unit + 2 * u);
        nseg = __ldcg(prm.ws_unit + 2 * u + 1);
        if (nseg <= 1) return;  // a whole unit: written by the decode kernel
    }
    const int g = col ? idx / D : 0, d = col ? idx % D : 0;
    const int s0 = first + u;
    float M = -CUDART_INF_F, Lsum = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = grp; p0 < nseg; p0 += 8 * MG) {
        float mp[8], lp[8];
        float4 op[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int p = p0 + i * MG;
            const bool in = col && p < nseg;
            const size_t s = static_cast<size_t>(s0 + p);
            mp[i] = in ? __ldcg(prm.ws_m + s * G + g) : -CUDART_INF_F;
            lp[i] = in ? __ldcg(prm.ws_l + s * G + g) : 0.f;
            op[i] = in ? __ldcg(reinterpret_cast<const float4 *>(prm.ws_o + (s * G + g) * D + d))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mc = M;
#pragma unroll
        for (int i = 0; i < 8; ++i) mc = fmaxf(mc, mp[i]);
        if (mc == -CUDART_INF_F) continue;
        const float a = exp2f(M - mc);  // 0 while M is still -inf
        O.x *= a;
        O.y *= a;
        O.z *= a;
        O.w *= a;
        Lsum *= a;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (mp[i] == -CUDART_INF_F) continue;  // a slice whose blocks were all skipped
            const float wt = exp2f(mp[i] - mc);
            O.x += wt * op[i].x;
            O.y += wt * op[i].y;
            O.z += wt * op[i].z;
            O.w += wt * op[i].w;
            Lsum += wt * lp[i];
        }
        M = mc;
    }
    float Lt = Lsum;
    float4 Ot = O;
    if constexpr (MG > 1) {
        sh_o[grp][lane] = O;
        sh_m[grp][lane] = M;
        sh_l[grp][lane] = Lsum;
        __syncthreads();
        if (grp != 0) return;
        float Mt = sh_m[0][lane];
#pragma unroll
        for (int w = 1; w < MG; ++w) Mt = fmaxf(Mt, sh_m[w][lane]);
        Lt = 0.f;
        Ot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < MG; ++w) {
            const float mw = sh_m[w][lane];
            if (mw == -CUDART_INF_F) continue;  // a warp with no slices, or only skipped ones
            const float wt = exp2f(mw - Mt);
            const float4 ow = sh_o[w][lane];
            Ot.x += wt * ow.x;
            Ot.y += wt * ow.y;
            Ot.z += wt * ow.z;
            Ot.w += wt * ow.w;
            Lt += wt * sh_l[w][lane];
        }
    }
    if (!col) return;
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
    Ot.x *= inv;
    Ot.y *= inv;
    Ot.z *= inv;
    Ot.w *= inv;
    store_out4(static_cast<T *>(prm.out) + (static_cast<size_t>(b) * prm.num_heads + hk * G + g) * D + d, Ot);
}

}  // namespace pa
