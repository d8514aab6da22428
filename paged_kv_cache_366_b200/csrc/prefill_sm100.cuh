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
// How it runs (bf16 in, fp32 accumulate, head_dim 128), warp-specialized:
//  * A CTA owns up to two Q tiles of 128 rows. Each row is one of (128 / G)
//    chunk tokens x the G query heads of one KV head (GQA packing), so every
//    K/V tile loaded serves all G heads of both Q tiles. A chunk too short to
//    reach the second tile (a decode token, a short verify chunk) runs one.
//  * Warp 0 streams Q and then 128-key K tiles by TMA with 128-byte swizzle
//    into a 2-stage ring, and warp 10 the V tiles into a 3-stage ring (2 over
//    an FP8 pool), so
//    neither load waits behind the other's free stage. A tile is eight 16-token
//    blocks, and each block of each 64-column half is one TMA box addressed
//    through the block table. Blocks past the context (and bad table entries) load from an
//    out-of-range row, which fills zeros. The producer zeroes the last tile's V
//    rows past the context before the MMA may read them (0 * NaN would poison O).
//  * Warp 1 issues the MMAs from one thread: S = Q K^T (M=128, N=128) and
//    O += P V (M=128, N=128, K=128), tcgen05.mma kind::f16, with S, P and O of
//    both Q tiles in tensor memory (512 columns). P is written as bf16 over the
//    first half of its own S and is the A operand of P V straight from tensor
//    memory. 128-key tiles keep the QK MMA at full rate (at N=64 it is bound by
//    shared-memory operand reads) and halve the hand-offs per key.
//  * The order per tile is PV(tile 0, j), QK(tile 0, j+1), PV(tile 1, j),
//    QK(tile 1, j+1): one Q tile's softmax overlaps the other tile's MMAs. A QK
//    overwrites P, so it waits for the P V before it (odone).
//  * A CTA with one Q tile and two or more K/V tiles splits: slot 1 (the second
//    S/O pair in TMEM and its softmax warps) runs the same queries over the odd
//    K/V tiles, slot 0 over the even ones, and the two (m, l, O) merge in the
//    epilogue (slot 1 hands m and l over in shared memory; slot 0 reads its O
//    from TMEM). Decode tokens and short verify chunks in a varlen batch then
//    keep two chains in flight per CTA without a second kernel.
//  * Warps 2..5 and 6..9 run the softmax of Q tiles 0 and 1; thread = row =
//    TMEM lane; a warp whose rows hold no chunk token only keeps the barrier
//    protocol. A thread reads its scores in two 64-key halves, masks keys past
//    its causal limit and computes p = 2^(s*scale*log2(e) - m) with one FMA
//    and one ex2, summing the fp32 p in packed pairs. The reference max m is
//    replaced (and O rescaled in TMEM) only when a row max grows by more than
//    2^8, so the first half is exponentiated before the second is read, and
//    only re-scaled in the rare case that the second half moves m.
//  * Over an FP8 (E4M3) pool the producers TMA-load each tile's codes into a
//    staging buffer and widen them exactly to f16 into the stage (one
//    cvt.rn.f16x2.e4m3x2 per pair), so the MMAs take f16 operands: q is
//    converted to f16 in shared memory once per CTA and P is written as f16.
//    k_scale joins the softmax scale and v_scale the output.
//  * Hand-offs are mbarriers only: full/empty per ring stage (empties committed
//    by tcgen05.commit), and per Q tile sfull (S ready; it also implies the
//    previous P V is done, so O may be rescaled), pready and odone. Every wait
//    is bounded and also gives up when another role has aborted. The MMA thread
//    drains its work before tensor memory is freed.
#pragma once

#include <cuda_fp16.h>
#include <math_constants.h>

#include <atomic>

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

// The eight K=16 steps of one tile's MMA, issued by one thread from one asm
// block. A shared-memory descriptor addresses 16-byte units in its low 14 bits,
// so the descriptor of base + off is the base's descriptor plus off / 16 (no
// carry below 256 KB): each step adds a constant instead of rebuilding both
// descriptors.

// S = Q K^T over head_dim 128: a and b describe the first step of Q and K
// (K-major, 128-byte swizzle, 64-column halves 16 KB apart; step kk advances
// (kk / 4) * 16 KB + (kk % 4) * 32 B). The first step overwrites S.
__device__ __forceinline__ void umma_qk_d128(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred pf, pt;\n\t.reg .b64 a1, b1;\n\t"
        "setp.ne.b32 pf, %3, %3;\n\t"
        "setp.eq.b32 pt, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, pf;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 b1, %2, 2;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, pt;\n\t"
        "add.s64 a1, %1, 4;\n\tadd.s64 b1, %2, 4;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, pt;\n\t"
        "add.s64 a1, %1, 6;\n\tadd.s64 b1, %2, 6;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, pt;\n\t"
        "add.s64 a1, %1, 1024;\n\tadd.s64 b1, %2, 1024;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, pt;\n\t"
        "add.s64 a1, %1, 1026;\n\tadd.s64 b1, %2, 1026;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, pt;\n\t"
        "add.s64 a1, %1, 1028;\n\tadd.s64 b1, %2, 1028;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, pt;\n\t"
        "add.s64 a1, %1, 1030;\n\tadd.s64 b1, %2, 1030;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, pt;\n\t"
        "}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc)
        : "memory");
}

// O (+)= P V over 128 keys: P, the A operand, is read from tensor memory (16
// keys = 8 columns per step); b describes V's first 16 keys (MN-major, 2 KB per
// 16 keys). The first step accumulates iff `accumulate`.
__device__ __forceinline__ void umma_pv_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred pa, pt;\n\t.reg .b32 a1;\n\t.reg .b64 b1;\n\t"
        "setp.ne.b32 pa, %4, 0;\n\t"
        "setp.eq.b32 pt, %3, %3;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, pa;\n\t"
        "add.s32 a1, %1, 8;\n\tadd.s64 b1, %2, 128;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, pt;\n\t"
        "add.s32 a1, %1, 16;\n\tadd.s64 b1, %2, 256;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, pt;\n\t"
        "add.s32 a1, %1, 24;\n\tadd.s64 b1, %2, 384;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, pt;\n\t"
        "add.s32 a1, %1, 32;\n\tadd.s64 b1, %2, 512;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, pt;\n\t"
        "add.s32 a1, %1, 40;\n\tadd.s64 b1, %2, 640;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, pt;\n\t"
        "add.s32 a1, %1, 48;\n\tadd.s64 b1, %2, 768;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, pt;\n\t"
        "add.s32 a1, %1, 56;\n\tadd.s64 b1, %2, 896;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, pt;\n\t"
        "}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
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

// 64 consecutive fp32 columns of this thread's TMEM lane, one load instruction.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, "
        "%36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, "
        "%57, %58, %59, %60, %61, %62, %63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
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

// Instruction descriptor, kind::f16: fp32 accumulator, A and B both bf16 or
// both f16, A K-major, B K-major (b_mn = 0) or MN-major (b_mn = 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16kind(int M, int N, int b_mn, bool f16) {
    return (1u << 4) | ((f16 ? 0u : 1u) << 7) | ((f16 ? 0u : 1u) << 10) | (static_cast<uint32_t>(b_mn) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---- geometry -------------------------------------------------------------------

constexpr int kPfWarps = 11;                 // K producer, MMA, 2 x 4 softmax warps, V producer
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kPfSoftmax0 = 2;               // first softmax warp
constexpr int kPfVWarp = 10;                 // the V producer
constexpr int kPfM = 128;                    // rows per Q tile (tokens x group heads)
constexpr int kPfNQ = 2;                     // Q tiles per CTA, ping-ponged
constexpr int kPfN = 128;                    // keys per K/V tile
constexpr int kPfD = 128;                    // head_dim
constexpr int kPfNSK = 2;                    // K pipeline stages
constexpr int kPfQHalf = kPfM * 64 * 2;      // a 64-column half of a Q tile: 16 KB
constexpr int kPfQTile = 2 * kPfQHalf;       // 32 KB
constexpr int kPfKVHalf = kPfN * 64 * 2;     // a 64-dim half of a K/V tile: 16 KB
constexpr int kPfKVTile = 2 * kPfKVHalf;     // 32 KB
constexpr int kPfOffQ = 0;
constexpr int kPfOffK = kPfOffQ + kPfNQ * kPfQTile;
constexpr int kPfTileBars = 3;  // per Q tile: sfull (S ready), pready (P written), odone (its P V done)

// Shared-memory layout. A bf16 pool streams V through three stages. An FP8
// (E4M3) pool streams it through two, and the room of the third holds the
// codes of one K tile and of one V tile as loaded, before the producer warps
// widen them to f16 into the stages the MMA reads.
template <bool FP8>
struct PfLayout {
    static constexpr int NSV = FP8 ? 2 : 3;  // V pipeline stages (a V tile is held longest)
    static constexpr int OffV = kPfOffK + kPfNSK * kPfKVTile;
    static constexpr int StgTile = kPfN * kPfD;  // E4M3 codes of one K or V tile: 16 KB
    static constexpr int OffStg = OffV + NSV * kPfKVTile;
    static constexpr int OffBar = OffStg + (FP8 ? 2 * StgTile : 0);
    // mbarriers: q, kfull[NSK], kempty[NSK], vfull[NSV], vempty[NSV], vzero, drain, the K and
    // the V staging buffers (FP8: codes landed), q converted to f16 (FP8), then kPfTileBars
    // per Q tile
    static constexpr int BarQ = 0, BarKF = 1, BarKE = BarKF + kPfNSK, BarVF = BarKE + kPfNSK, BarVE = BarVF + NSV,
                         BarVZ = BarVE + NSV, BarDrain = BarVZ + 1, BarStg = BarDrain + 1, BarQC = BarStg + 2,
                         BarTile = BarQC + 1, Bars = BarTile + kPfTileBars * kPfNQ;
    static constexpr int OffSlot = OffBar + Bars * 8;  // TMEM base address, abort flag
    static constexpr int OffML = OffSlot + 16;         // (m, l) of slot 1 per row, for the split merge
    static constexpr int Smem = OffML + 2 * kPfM * 4 + 1024;  // + room to align the base to 1024 B
    static_assert(Smem <= 232448, "prefill shared memory over the 227 KB limit");
    static_assert(OffStg % 1024 == 0 && StgTile % 1024 == 0, "staging and stages stay 1024-byte aligned");
};
// Tensor memory columns: S_A, S_B (128 fp32 each), then O_A, O_B (128 each). P of
// a Q tile (128 bf16 = 64 columns) overwrites the first half of its own S.
constexpr uint32_t kPfColP = 0;
constexpr uint32_t kPfColO = kPfNQ * kPfN;
constexpr uint32_t kPfTmemCols = 512;
constexpr int kPfBlocksPerTile = kPfN / kBlockSize;  // 8
static_assert(kPfColO + kPfNQ * kPfD <= kPfTmemCols, "tensor memory over 512 columns");
static_assert(kPfBlocksPerTile <= 32, "one producer lane per block of a tile");

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
    int num_seqs;
    float scale_log2;  // softmax scale * log2(e) (times k_scale for an FP8 cache)
    float v_scale;     // 1, or the FP8 value scale
};

// max(a, b, c) in one instruction (sm_100 has a three-input max)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Two probabilities as the PV MMA's A operand: a bf16 pair, or an f16 pair
// (F16), the first in the low half; and back.
template <bool F16>
__device__ __forceinline__ uint32_t pack_p(float p0, float p1) {
    if constexpr (F16) {
        const __half2 h = __floats2half2_rn(p0, p1);
        return *reinterpret_cast<const uint32_t *>(&h);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
}
template <bool F16>
__device__ __forceinline__ void unpack_p(uint32_t u, float &p0, float &p1) {
    if constexpr (F16) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&u));
        p0 = f.x;
        p1 = f.y;
    } else {
        p0 = __uint_as_float(u << 16);
        p1 = __uint_as_float(u & 0xffff0000u);
    }
}

// p = 2^(x * sc + nm) for 64 scores of one row: the fp32 p are summed into acc
// in packed pairs, and the bf16 (F16: f16) pairs (keys 2w, 2w+1 in column w) are
// stored to 32 TMEM columns at taddr.
template <bool F16>
__device__ __forceinline__ void pf_exp_half(const float (&x)[64], float sc, float nm, f32x2 (&acc)[4],
                                            uint32_t taddr) {
    float pv[32];
#pragma unroll
    for (int w = 0; w < 32; ++w) {
        f32x2 arg = pack2(nm, nm);  // x * sc + nm for the pair, one packed FMA
        fma2(arg, pack2(x[2 * w], x[2 * w + 1]), pack2(sc, sc));
        float a0, a1;
        unpack2(arg, a0, a1);
        const float p0 = ex2_approx(a0);
        const float p1 = ex2_approx(a1);
        add2(acc[w & 3], pack2(p0, p1));
        pv[w] = __uint_as_float(pack_p<F16>(p0, p1));
    }
    // finish the sums here: otherwise the compiler keeps the 64 p values alive
    // into the next half and runs out of registers
    asm volatile("" : "+l"(acc[0]), "+l"(acc[1]), "+l"(acc[2]), "+l"(acc[3]));
    tmem_st32(taddr, pv);
}

// Lines to keep in L2 over others (createpolicy result).
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Four E4M3 codes (low byte = element 0) to four f16 values, exactly (every
// E4M3 value, subnormals included, is a normal f16 value or zero): two f16
// pairs, element 0 in the low half of the first. One conversion per pair.
__device__ __forceinline__ uint2 e4m3x4_to_f16x4(uint32_t w) {
    uint32_t lo, hi;
    asm("{\n\t.reg .b16 c;\n\t"
        "cvt.u16.u32 c, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, c;\n\t"
        "cvt.u16.u32 c, %3;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, c;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w & 0xffffu), "r"(w >> 16));
    return make_uint2(lo, hi);
}

// A bf16 pair to an f16 pair, rounded to nearest (exact for magnitudes in f16's
// normal range and for zero).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u) {
    const __half2 h = __floats2half2_rn(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Work slots of a varlen launch: sequence b owns the slots starting at
// S_b = cu_q_lens[b] / per_cta + b (per_cta = chunk tokens one CTA covers), and
// uses the first ceil(q_len_b / per_cta) of them. S is strictly increasing and
// S_{b+1} - S_b >= ceil(q_len_b / per_cta), so num_q_tokens / per_cta + num_seqs
// slots cover every sequence and at most one slot per sequence stays empty (a
// grid of max tiles x sequences would leave most decode-token CTAs empty).
// Returns the largest b with S_b <= w: each step the warp probes 32 evenly spaced
// candidates and keeps the interval after the last one at or below w.
__device__ __forceinline__ int pf_find_seq(const int *cu_q_lens, int num_seqs, int per_cta, int w, int lane) {
    int lo = 0, hi = num_seqs;  // S_lo <= w (S_0 = 0); the answer lies in [lo, hi)
    while (hi - lo > 1) {
        const int step = (hi - lo + 31) / 32;
        const int cand = lo + lane * step;
        const bool le = cand < hi && __ldg(cu_q_lens + cand) / per_cta + cand <= w;
        const unsigned m = __ballot_sync(0xffffffffu, le);
        const int last = m ? 31 - __clz(m) : 0;
        lo += last * step;
        hi = min(hi, lo + step);
    }
    return lo;
}

// Compile-time tag for the split and unsplit copies of the kernel's roles.
template <bool B>
struct PfSplit {
    static constexpr bool value = B;
};

// Bounded mbarrier wait that also gives up when another role of the CTA has aborted.
__device__ __forceinline__ bool pf_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            flag_status(PA_STATUS_WAIT_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// FP8: the caches hold E4M3 codes (values code * k_scale, code * v_scale);
// q and out stay bf16.
template <int G, bool FP8>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const PrefillParams prm, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    using L = PfLayout<FP8>;
    constexpr int TOK = kPfM / G;  // chunk tokens per Q tile
    constexpr int PER_CTA = kPfNQ * TOK;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    // grid.x = slots x KV heads, KV head fastest, so the slots of one chunk (its
    // longest tile pairs first) start together
    const int hk = static_cast<int>(blockIdx.x % static_cast<unsigned>(prm.num_kv_heads));
    const int w = static_cast<int>(blockIdx.x / static_cast<unsigned>(prm.num_kv_heads));

    // Launched as a programmatic dependent: wait for the previous kernel (e.g. the
    // cache write of this chunk) before reading any input.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- this CTA's sequence and tile pair (every warp finds the same) ----
    const int b = pf_find_seq(prm.cu_q_lens, prm.num_seqs, PER_CTA, w, lane);
    const int q0 = __ldg(prm.cu_q_lens + b), q1 = __ldg(prm.cu_q_lens + b + 1);
    const int slot = w - (q0 / PER_CTA + b);  // 0 .. of this sequence's slots
    const int q_len = q1 - q0;
    const int c = __ldg(prm.context_lens + b);
    const bool first = slot == 0 && hk == 0 && tid == 0;
    if (q_len < 0 || q_len > c || q1 > prm.num_q_tokens) {
        if (first) flag_status(PA_STATUS_BAD_QUERY);
        return;
    }
    if (c > prm.max_blocks_per_seq * kBlockSize) {
        if (first) flag_status(PA_STATUS_BAD_CONTEXT);
        return;
    }
    const int n_ct = (q_len + PER_CTA - 1) / PER_CTA;
    if (slot >= n_ct) return;
    const int ct = n_ct - 1 - slot;  // longest tile pairs first
    const int t0 = ct * kPfNQ * TOK;
    const int n_q = q_len - t0 > TOK ? 2 : 1;  // Q tiles holding chunk tokens (a short chunk uses one)
    const int o = c - q_len;
    const int kv_end = o + min(t0 + n_q * TOK, q_len);  // keys needed: [0, kv_end)
    const int n_tiles = (kv_end + kPfN - 1) / kPfN;
    // Split: a CTA with one Q tile and two or more K/V tiles runs the second slot
    // (its TMEM, its softmax warps) on the same queries over the odd K/V tiles,
    // the first slot takes the even ones, and the two (m, l, O) merge at the end.
    // Decode tokens and short verify chunks then keep two chains in flight.
    const bool split_cta = n_q == 1 && n_tiles >= 2;
    const int nblk_seq = (c + kBlockSize - 1) / kBlockSize;
    const bool zero_tail = n_tiles * kPfN > c;  // the last tile holds keys past the context

    // ---- shared memory (base aligned to 1024 B for the 128-byte swizzle) ----
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    unsigned char *base = smem_raw + (base_s - raw_s);
    const uint32_t bars = base_s + L::OffBar;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L::OffSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + L::OffSlot + 4);

    if (tid == 0) {
        mbar_init(bar(L::BarQ), 1);
        for (int i = 0; i < kPfNSK; ++i) {
            mbar_init(bar(L::BarKF + i), 1);
            mbar_init(bar(L::BarKE + i), 1);
        }
        for (int i = 0; i < L::NSV; ++i) {
            mbar_init(bar(L::BarVF + i), 1);
            mbar_init(bar(L::BarVE + i), 1);
        }
        mbar_init(bar(L::BarVZ), 1);
        mbar_init(bar(L::BarDrain), 1);
        mbar_init(bar(L::BarStg), 1);      // FP8: K codes landed in the staging buffer
        mbar_init(bar(L::BarStg + 1), 1);  // FP8: V codes landed
        mbar_init(bar(L::BarQC), 2);  // FP8: both producer warps have converted their Q tile to f16
        for (int qi = 0; qi < kPfNQ; ++qi) {
            mbar_init(bar(L::BarTile + kPfTileBars * qi + 0), 1);    // sfull: MMA commit
            mbar_init(bar(L::BarTile + kPfTileBars * qi + 1), 128);  // pready: every softmax thread of the slot
            mbar_init(bar(L::BarTile + kPfTileBars * qi + 2), 1);    // odone: MMA commit
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_addr(tmem_slot), kPfTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // The roles are compiled twice, split and unsplit, and each CTA runs one copy:
    // a runtime flag in the inner loops cost the unsplit prefill about 10 %.
    auto roles = [&](auto split_tag) {
        constexpr bool split = decltype(split_tag)::value;
        const int n_slots = split ? 2 : n_q;
        if (warp == 0 || warp == kPfVWarp) {
            // ====== producers: warp 0 loads Q and the K tiles, the V warp the V tiles (TMA) ======
            // Separate rings let a K tile load as soon as its stage is free, whatever V waits on.
            const bool is_v = warp == kPfVWarp;
            const int *trow = prm.block_tables + static_cast<size_t>(b) * prm.max_blocks_per_seq;
            const int oob_row = static_cast<int>(prm.num_blocks * kBlockSize);  // past the pool: TMA fills zeros
            auto tile_row = [&](int t) -> int {  // pool row of block `lane` of tile t
                if (lane >= kPfBlocksPerTile || t >= n_tiles) return oob_row;
                const int lb = t * kPfBlocksPerTile + lane;
                if (lb >= nblk_seq) return oob_row;
                const int pb = __ldg(trow + lb);
                if (pb < 0 || pb >= prm.num_blocks) {
                    flag_status(PA_STATUS_BAD_BLOCK_ID);
                    return oob_row;
                }
                return pb * kBlockSize;
            };
            const CUtensorMap *tm = is_v ? &tm_v : &tm_k;
            const int ns = is_v ? L::NSV : kPfNSK;
            const uint32_t ring = base_s + (is_v ? L::OffV : kPfOffK);
            const int b_full = is_v ? L::BarVF : L::BarKF, b_empty = is_v ? L::BarVE : L::BarKE;
            auto load_tile = [&](int s, int row) {
                const uint32_t full = bar(b_full + s);
                if (lane == 0) mbar_arrive_expect_tx(full, kPfKVTile);
                __syncwarp();
                if (lane < kPfBlocksPerTile) {
                    const uint32_t d = ring + s * kPfKVTile + lane * (kBlockSize * 128);  // 16 rows of 128 B
                    tma_load_3d(d, tm, 0, hk, row, full);
                    tma_load_3d(d + kPfKVHalf, tm, 64, hk, row, full);
                }
            };
            if (!is_v && lane == 0) {
                mbar_arrive_expect_tx(bar(L::BarQ), n_q * kPfQTile);
                for (int qi = 0; qi < n_q; ++qi) {
                    const uint32_t dq = base_s + kPfOffQ + qi * kPfQTile;
                    const int qrow = q0 + t0 + qi * TOK;
                    tma_load_3d(dq, &tm_q, 0, hk * G, qrow, bar(L::BarQ));
                    tma_load_3d(dq + kPfQHalf, &tm_q, 64, hk * G, qrow, bar(L::BarQ));
                }
            }
            if constexpr (FP8) {
                // The E4M3 codes of tile j land by TMA in this warp's staging buffer (16 rows
                // x 128 B per block, row-major). The warp widens them to f16 into stage s, in
                // the 128-byte-swizzled layout a TMA load of a 16-bit tile leaves (16-byte
                // chunk k of row r at chunk k ^ (r % 8)), arrives on the stage's full barrier,
                // and sends the next tile's codes, which load while the MMA works.
                const uint32_t stg = base_s + L::OffStg + (is_v ? L::StgTile : 0);
                const unsigned char *stg_p = base + L::OffStg + (is_v ? L::StgTile : 0);
                const uint32_t b_stg = bar(L::BarStg + (is_v ? 1 : 0));
                auto load_codes = [&](int rows) {  // this lane's block of the tile (lanes < 8)
                    if (lane == 0) mbar_arrive_expect_tx(b_stg, L::StgTile);
                    __syncwarp();
                    // evict-last: the other CTAs of the chunk read the same codes (measured
                    // 1.2 % faster on a 2048-token chunk than the default policy)
                    if (lane < kPfBlocksPerTile)
                        tma_load_3d_policy(stg + lane * (kBlockSize * 128), tm, 0, hk, rows, b_stg, policy_evict_last());
                };
                int loaded = 1;  // code tiles sent to the staging buffer
                load_codes(tile_row(0));
                // while the first codes load: q to f16 in place (the MMAs take f16 operands
                // here), Q tile 0 by the K producer, Q tile 1 (if any) by the V producer
                const int qt = is_v ? 1 : 0;
                if (qt < n_q) {
                    const bool qok = __all_sync(0xffffffffu, pf_wait(bar(L::BarQ), 0, abort_flag));
                    if (qok) {
                        unsigned char *qp = base + kPfOffQ + qt * kPfQTile;
#pragma unroll 4
                        for (int i = lane; i < kPfQTile / 16; i += 32) {
                            uint4 w = *reinterpret_cast<const uint4 *>(qp + i * 16);
                            w = make_uint4(bf16x2_to_f16x2(w.x), bf16x2_to_f16x2(w.y), bf16x2_to_f16x2(w.z),
                                           bf16x2_to_f16x2(w.w));
                            *reinterpret_cast<uint4 *>(qp + i * 16) = w;
                        }
                        fence_async_smem();  // the converted q to the MMA's proxy
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::BarQC));
                bool ok = true;
                for (int j = 0; j < n_tiles && ok; ++j) {
                    const int s = j % ns, u = j / ns;
                    const int row_next = tile_row(j + 1);
                    ok = pf_wait(b_stg, j & 1, abort_flag);
                    if (ok && u >= 1) ok = pf_wait(bar(b_empty + s), (u - 1) & 1, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    // V rows past the context may hold any code (NaN included), and 0 * NaN
                    // would poison O: they are written as zeros
                    const int valid = is_v ? c - j * kPfN : kPfN;
                    unsigned char *dst = base + (is_v ? L::OffV : kPfOffK) + s * kPfKVTile;
#pragma unroll 4
                    for (int it = 0; it < kPfN * 8 / 32; ++it) {
                        const int i = it * 32 + lane, r = i / 8, c16 = i % 8;  // row r, codes 16 c16 .. + 15
                        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
                        if (r < valid) {
                            const uint4 w = *reinterpret_cast<const uint4 *>(stg_p + r * 128 + c16 * 16);
                            const uint2 x0 = e4m3x4_to_f16x4(w.x), x1 = e4m3x4_to_f16x4(w.y);
                            const uint2 x2 = e4m3x4_to_f16x4(w.z), x3 = e4m3x4_to_f16x4(w.w);
                            lo = make_uint4(x0.x, x0.y, x1.x, x1.y);
                            hi = make_uint4(x2.x, x2.y, x3.x, x3.y);
                        }
                        // dims 16 c16 .. + 15 are chunks 2 c16 % 8 and + 1 of half c16 / 4
                        unsigned char *rp = dst + (c16 / 4) * kPfKVHalf + r * 128;
                        const int k8 = (2 * c16) & 7;
                        *reinterpret_cast<uint4 *>(rp + ((k8 ^ (r & 7)) * 16)) = lo;
                        *reinterpret_cast<uint4 *>(rp + (((k8 + 1) ^ (r & 7)) * 16)) = hi;
                    }
                    // the widened tile to the MMA's (async) proxy, and the staging reads
                    // ordered before the next TMA load overwrites the codes
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(b_full + s));
                    if (j + 1 < n_tiles) {
                        load_codes(row_next);
                        loaded = j + 2;
                    }
                }
                // a code load nobody widened lands before the CTA exits
                if (*abort_flag) mbar_wait(b_stg, (loaded - 1) & 1);
            } else {
                int row = tile_row(0);
                int issued = 0;
                bool ok = true;
                for (int j = 0; j < n_tiles && ok; ++j) {
                    const int s = j % ns, u = j / ns;
                    const int row_next = tile_row(j + 1);  // fetched while this tile's loads go out
                    if (u >= 1) ok = pf_wait(bar(b_empty + s), (u - 1) & 1, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    load_tile(s, row);
                    issued = j + 1;
                    if (is_v && j == n_tiles - 1 && zero_tail) {
                        // keys past the context: their V rows (tail slots) may hold anything, and
                        // 0 * NaN would poison O, so zero them before the MMA reads the tile
                        ok = __all_sync(0xffffffffu, pf_wait(bar(b_full + s), u & 1, abort_flag));
                        if (ok) {
                            const int first_bad = max(0, c - j * kPfN);
                            unsigned char *vt = base + L::OffV + s * kPfKVTile;
                            for (int i = lane; i < (kPfN - first_bad) * 16; i += 32) {
                                const int r = first_bad + i / 16, half = (i / 8) & 1, chunk = i & 7;
                                *reinterpret_cast<uint4 *>(vt + half * kPfKVHalf + r * 128 + chunk * 16) =
                                    make_uint4(0, 0, 0, 0);
                            }
                            fence_async_smem();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar(L::BarVZ));
                        }
                    }
                    row = row_next;
                }
                if (*abort_flag) {  // let loads nobody consumed land before the CTA exits
                    for (int i = 0; i < issued; ++i) mbar_wait(bar(b_full + i % ns), (i / ns) & 1);
                }
            }
        } else if (warp == 1) {
            // ================= MMA issue (one thread) =================
            if (lane == 0) {
                // an FP8 pool's tiles are widened to f16, so its MMAs take f16 operands
                constexpr uint32_t kIdQK = idesc_f16kind(kPfM, kPfN, 0, FP8);
                constexpr uint32_t kIdPV = idesc_f16kind(kPfM, kPfD, 1, FP8);
                auto b_tile = [&](int qi, int k) -> uint32_t { return bar(L::BarTile + kPfTileBars * qi + k); };
                // slot qi takes K/V tiles tile_of(qi, 0 .. n_of(qi) - 1); `last` marks the
                // slot after whose MMA a K/V stage may be refilled
                auto n_of = [&](int qi) -> int { return split ? (n_tiles - qi + 1) / 2 : n_tiles; };
                auto tile_of = [&](int qi, int i) -> int { return split ? 2 * i + qi : i; };
                const auto last = [&](int qi) -> bool { return split || qi == n_q - 1; };
                auto issue_qk = [&](int qi, int j) {  // S_qi = Q K_j^T
                    const uint32_t qb = base_s + kPfOffQ + (split ? 0 : qi) * kPfQTile;
                    const uint32_t kb = base_s + kPfOffK + (j % kPfNSK) * kPfKVTile;
                    static_assert(kPfQHalf == 16384 && kPfKVHalf == 16384 && kPfD == 128, "umma_qk_d128 steps");
                    umma_qk_d128(tmem + qi * kPfN, smem_desc_sw128(qb, 16, 1024), smem_desc_sw128(kb, 16, 1024),
                                 kIdQK);
                    umma_commit(b_tile(qi, 0));
                    if (last(qi)) umma_commit(bar(L::BarKE + j % kPfNSK));
                };
                auto issue_pv = [&](int qi, int j, bool acc) {  // O_qi (+)= P_qi V_j, P read from tensor memory
                    const uint32_t pt = tmem + qi * kPfN + kPfColP;
                    const uint32_t vb = base_s + L::OffV + (j % L::NSV) * kPfKVTile;
                    static_assert(kPfN == 128, "umma_pv_k128 covers 128 keys");
                    umma_pv_k128(tmem + kPfColO + qi * kPfD, pt, smem_desc_sw128(vb, kPfKVHalf, 1024), kIdPV,
                                 acc ? 1u : 0u);
                    umma_commit(b_tile(qi, 2));
                    if (last(qi)) umma_commit(bar(L::BarVE + j % L::NSV));
                };
                // the first slot to read a K/V tile waits for it; in the unsplit order the
                // second slot's MMA on the same tile comes after the first one's
                auto wait_k = [&](int qi, int j) {
                    return (qi > 0 && !split) || pf_wait(bar(L::BarKF + j % kPfNSK), (j / kPfNSK) & 1, abort_flag);
                };
                auto wait_v = [&](int qi, int j) {
                    if (qi > 0 && !split) return true;
                    // a bf16 pool's last tile is ready once its tail rows are zeroed; an FP8
                    // pool's producer zeroes them while it widens the codes
                    return (!FP8 && j == n_tiles - 1 && zero_tail)
                               ? pf_wait(bar(L::BarVZ), 0, abort_flag)
                               : pf_wait(bar(L::BarVF + j % L::NSV), (j / L::NSV) & 1, abort_flag);
                };
                bool ok = pf_wait(bar(FP8 ? L::BarQC : L::BarQ), 0, abort_flag);
                for (int qi = 0; qi < n_slots && ok; ++qi) {
                    ok = wait_k(qi, tile_of(qi, 0));
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk(qi, tile_of(qi, 0));
                }
                const int rounds = n_of(0);
                for (int i = 0; i < rounds && ok; ++i) {
                    for (int qi = 0; qi < n_slots && ok; ++qi) {
                        if (i >= n_of(qi)) continue;
                        const int j = tile_of(qi, i);
                        // O += P V once softmax qi has written P (and rescaled O)
                        ok = pf_wait(b_tile(qi, 1), i & 1, abort_flag) && wait_v(qi, j);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(qi, j, i > 0);
                        if (i + 1 >= n_of(qi)) continue;
                        // the next S overwrites P: wait for this P V to finish reading it
                        const int j1 = tile_of(qi, i + 1);
                        ok = pf_wait(b_tile(qi, 2), i & 1, abort_flag) && wait_k(qi, j1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_qk(qi, j1);
                    }
                }
                // every MMA issued so far completes before tensor memory can be freed
                umma_commit(bar(L::BarDrain));
                mbar_wait(bar(L::BarDrain), 0);
            }
            __syncwarp();
        } else {
            // ====== softmax: warps 2..5 run slot 0, warps 6..9 slot 1; thread = row = TMEM lane ======
            const int qi = (warp - kPfSoftmax0) / 4;
            const int quad = warp & 3;  // a warp reaches TMEM lanes 32 * (warp % 4) .. + 31
            const int r = quad * 32 + lane;
            const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
            const uint32_t tS = tmem + qi * kPfN + lane_base, tO = tmem + kPfColO + qi * kPfD + lane_base;
            const uint32_t b_sfull = bar(L::BarTile + kPfTileBars * qi + 0);
            const uint32_t b_pready = bar(L::BarTile + kPfTileBars * qi + 1);
            const uint32_t b_odone = bar(L::BarTile + kPfTileBars * qi + 2);
            const int tq = t0 + (split ? 0 : qi) * TOK;  // first chunk token of this slot's queries
            const int n_mine = split ? (n_tiles - qi + 1) / 2 : n_tiles;  // K/V tiles of this slot
            const int rows_valid = max(0, min(TOK, q_len - tq));
            // warps whose 32 rows hold no chunk token only keep the barrier protocol
            const bool active = (quad * 32) / G < rows_valid;
            const int tok = min(tq + r / G, q_len - 1);  // rows past the chunk reuse the last token's limit
            const int pos = o + tok;                      // causal limit: keys 0..pos
            float m_ref = -CUDART_INF_F, l_sum = 0.f;
            bool ok = qi < n_slots;
            for (int i = 0; i < n_mine && ok; ++i) {
                const int j = split ? 2 * i + qi : i;  // K/V tile
                ok = __all_sync(0xffffffffu, pf_wait(b_sfull, i & 1, abort_flag));
                if (!ok) break;
                if (active) {
                    tc_fence_after();
                    // Scores in two 64-key halves a (keys 0..63) and b (64..127), raw q.k; the
                    // scale (> 0) is applied inside the exponent. Half a is exponentiated
                    // against the reference max as it stands after a, and its P goes over
                    // S columns 0..31 (already read). If half b then raises that max (rare
                    // once a row has warmed up), P of a and its sum are scaled down to the
                    // new max. P of b goes over columns 32..63.
                    const int key0 = j * kPfN;
                    const bool edge = key0 + kPfN - 1 > pos;
                    const float sl2 = prm.scale_log2;
                    float h[64];
                    auto load_half = [&](int half) {  // scores of keys key0 + 64*half .. + 63, masked
                        tmem_ld64(tS + 64 * half, h);
                        if (edge) {
#pragma unroll
                            for (int i = 0; i < 64; ++i)
                                if (key0 + 64 * half + i > pos) h[i] = -CUDART_INF_F;
                        }
                    };
                    auto half_max = [&]() -> float {  // three-input max: two new scores per instruction
                        float m8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(h[i], h[i + 8]);
#pragma unroll
                        for (int i = 16; i < 64; i += 16)
#pragma unroll
                            for (int k = 0; k < 8; ++k) m8[k] = fmax3(m8[k], h[i + k], h[i + 8 + k]);
                        return fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) *
                               sl2;
                    };
                    auto raise = [&](float mx) -> float {  // lazy: move the max only past a 2^8 margin
                        if (!(mx > m_ref + 8.f)) return 1.f;
                        const float f = m_ref == -CUDART_INF_F ? 0.f : exp2f(m_ref - mx);
                        m_ref = mx;
                        return f;
                    };
                    auto exp_half = [&](f32x2 (&sum)[4], uint32_t col) {
                        // no unmasked key yet (m = -inf): every p is 0
                        pf_exp_half<FP8>(h, sl2, m_ref == -CUDART_INF_F ? -CUDART_INF_F : -m_ref, sum, tS + col);
                    };
                    f32x2 acc_a[4] = {0ull, 0ull, 0ull, 0ull}, acc[4] = {0ull, 0ull, 0ull, 0ull};
                    load_half(0);
                    float alpha = raise(half_max());  // factor for O and l of the earlier tiles
                    exp_half(acc_a, 0);
                    load_half(1);
                    const float beta = raise(half_max());  // factor for half a of this tile
                    if (__any_sync(0xffffffffu, beta != 1.f)) {
                        float pa[32];
                        tmem_ld32(tS, pa);
#pragma unroll
                        for (int w = 0; w < 32; ++w) {
                            float p0, p1;
                            unpack_p<FP8>(__float_as_uint(pa[w]), p0, p1);
                            pa[w] = __uint_as_float(pack_p<FP8>(p0 * beta, p1 * beta));
                        }
                        tmem_st32(tS, pa);
                        const f32x2 b2 = pack2(beta, beta);
#pragma unroll
                        for (int e = 0; e < 4; ++e) mul2(acc_a[e], b2);
                        alpha *= beta;
                    }
                    exp_half(acc, 32);
                    // O of the earlier tiles takes the same factor as l. S of this tile is
                    // complete, and so is every earlier MMA (the P V of tile j-1
                    // included), so O is stable here.
                    if (i > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {  // tcgen05.ld/st are warp-collective
#pragma unroll 1
                        for (int ch = 0; ch < kPfD / 32; ++ch) {
                            float v[32];
                            tmem_ld32(tO + ch * 32, v);
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] *= alpha;
                            tmem_st32(tO + ch * 32, v);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) add2(acc[e], acc_a[e]);
                    add2(acc[0], acc[1]);
                    add2(acc[2], acc[3]);
                    add2(acc[0], acc[2]);
                    float lo, hi;
                    unpack2(acc[0], lo, hi);
                    l_sum = l_sum * alpha + (lo + hi);
                    tc_fence_before();  // P and O visible to the MMA issued after the barrier
                }
                mbar_arrive(b_pready);
            }
            // ---- epilogue: out = O / l for the valid rows; a split CTA first merges slot 1 ----
            if (ok && active) ok = __all_sync(0xffffffffu, pf_wait(b_odone, (n_mine - 1) & 1, abort_flag));
            float wa = 1.f, wb = 0.f;  // weights of this slot's and of slot 1's (O, l)
            if (split) {
                // slot 1 hands (m, l) to slot 0 through shared memory; its O stays in TMEM,
                // where slot 0's warps (same TMEM lanes) read it. All 8 softmax warps meet here.
                float *ml = reinterpret_cast<float *>(base + L::OffML);
                if (qi == 1) {
                    ml[r] = m_ref;
                    ml[kPfM + r] = l_sum;
                }
                tc_fence_before();
                asm volatile("bar.sync 1, %0;" ::"n"(8 * 32) : "memory");
                tc_fence_after();
                if (qi == 0) {
                    const float mb = ml[r], lb = ml[kPfM + r];
                    const float mm = fmaxf(m_ref, mb);
                    wa = m_ref == -CUDART_INF_F ? 0.f : exp2f(m_ref - mm);
                    wb = mb == -CUDART_INF_F ? 0.f : exp2f(mb - mm);
                    l_sum = wa * l_sum + wb * lb;
                }
            }
            if (ok && active && (qi == 0 || !split)) {
                tc_fence_after();
                const bool row_ok = r / G < rows_valid;
                const float inv = l_sum > 0.f ? prm.v_scale / l_sum : 0.f;
                const float ia = wa * inv, ib = wb * inv;
                const uint32_t tOb = tmem + kPfColO + kPfD + lane_base;  // O of slot 1 (split only)
                const int orow = row_ok ? q0 + tq + r / G : q0;
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(prm.out) +
                                     (static_cast<size_t>(orow) * prm.num_heads + hk * G + r % G) * kPfD;
#pragma unroll 1
                for (int ch = 0; ch < kPfD / 32; ++ch) {  // 32 columns at a time bounds registers
                    float v[32];
                    tmem_ld32(tO + ch * 32, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= ia;
                    if (split) {
                        float vb[32];
                        tmem_ld32(tOb + ch * 32, vb);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = fmaf(vb[i], ib, v[i]);
                    }
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 pkt;
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(v[i], v[i + 1]);
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[i + 4], v[i + 5]);
                        __nv_bfloat162 h3 = __floats2bfloat162_rn(v[i + 6], v[i + 7]);
                        pkt.x = *reinterpret_cast<uint32_t *>(&h0);
                        pkt.y = *reinterpret_cast<uint32_t *>(&h1);
                        pkt.z = *reinterpret_cast<uint32_t *>(&h2);
                        pkt.w = *reinterpret_cast<uint32_t *>(&h3);
                        if (row_ok) *reinterpret_cast<uint4 *>(dst + ch * 32 + i) = pkt;
                    }
                }
            }
            tc_fence_before();
        }
    };
    if (split_cta)
        roles(PfSplit<true>{});
    else
        roles(PfSplit<false>{});
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

template <int G, bool FP8>
int launch_prefill_g(const PrefillParams &prm, const void *q, const void *k_cache, const void *v_cache,
                     int num_seqs, int max_q_len, int num_q_tokens, const pa_shape *s, cudaStream_t st) {
    constexpr int TOK = kPfM / G;
    CUtensorMap tm_q{}, tm_k{}, tm_v{};
    const uint64_t rows = static_cast<uint64_t>(s->num_blocks) * kBlockSize;
    using L = PfLayout<FP8>;
    // K/V boxes: a block's 16 rows of one KV head; bf16 as two 64-dim halves with the
    // 128-byte swizzle the MMA reads, FP8 codes as whole 128-byte rows for the widening
    const int ce = FP8 ? 1 : 2;
    const uint32_t bx = FP8 ? kPfD : 64;
    const CUtensorMapSwizzle sw = FP8 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B;
    if (!encode_3d(&tm_q, q, kPfD, s->num_heads, num_q_tokens, 2, 64, G, TOK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_3d(&tm_k, k_cache, kPfD, s->num_kv_heads, rows, ce, bx, 1, kBlockSize, sw) ||
        !encode_3d(&tm_v, v_cache, kPfD, s->num_kv_heads, rows, ce, bx, 1, kBlockSize, sw))
        return PA_ERR_UNSUPPORTED;
    // the shared-memory opt-in, once per device (bit per device; safe across host threads)
    static std::atomic<uint64_t> attr_done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    const uint64_t bit = uint64_t{1} << (dev & 63);
    if (!(attr_done.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(prefill_kernel<G, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::Smem) !=
            cudaSuccess)
            return PA_ERR_CUDA;
        attr_done.fetch_or(bit, std::memory_order_acq_rel);
    }
    const long long slots = static_cast<long long>(num_q_tokens) / (kPfNQ * TOK) + num_seqs;
    if (slots * s->num_kv_heads > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
    (void)max_q_len;  // the slot grid covers every chunk whatever its length
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(slots * s->num_kv_heads), 1, 1);
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = L::Smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_kernel<G, FP8>, prm, tm_q, tm_k, tm_v) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

inline int launch_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *cu_q_lens,
                          const int32_t *context_lens, int32_t num_seqs, int32_t max_q_len, int32_t num_q_tokens,
                          float scale, const pa_shape *s, cudaStream_t st) {
    if (num_seqs < 1) return PA_ERR_INVALID_ARGUMENT;
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
    prm.num_seqs = num_seqs;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.v_scale = 1.f;
    if (s->kv_fp8) {  // K = code * k_scale goes into the exponent's scale, V = code * v_scale into O's
        prm.scale_log2 *= s->k_scale;
        prm.v_scale = s->v_scale;
    }
#define PA_PREFILL_G(g)                                                                                           \
    case g:                                                                                                       \
        return s->kv_fp8                                                                                          \
                   ? launch_prefill_g<g, true>(prm, q, k_cache, v_cache, num_seqs, max_q_len, num_q_tokens, s, st) \
                   : launch_prefill_g<g, false>(prm, q, k_cache, v_cache, num_seqs, max_q_len, num_q_tokens, s, st);
    switch (s->num_heads / s->num_kv_heads) {
        PA_PREFILL_G(1)
        PA_PREFILL_G(2)
        PA_PREFILL_G(4)
        PA_PREFILL_G(8)
        default: return PA_ERR_UNSUPPORTED;
    }
#undef PA_PREFILL_G
}

}  // namespace pa
