// tcgen05 (5th-generation tensor core) kernel of the FLARE++ mixer backward,
// 16-bit I/O (bf16 or fp16).
//
// Every backward step of the three attentions O = softmax_rows(scale A B^T) C
// of the FLARE.py README's FLARE++ block has the same shape when written per
// tile: a [128 x D] row tile (A for the scores, C for the output-gradient
// products) against a stream of [KT x D] column tiles (B, and E), with
//     S  = A B^T                        score
//     dP = C E^T                        <dO_r, C_j> (or its transposed form)
//     P  = 2^(scale log2(e) S - lse)    softmax weight, from the forward's log-sum-exp
//     dS = P (dP - Delta)               gradient of the score
//     acc1 += dS B                      (M=128, N=D, K=KT: A = dS from TMEM)
//     acc2 += P E                       (optional; A = P from TMEM)
// where lse and Delta belong either to the row (the softmax runs along the
// columns: the row-side gradients) or to the column (the softmax runs along
// the rows: the column-side gradients).  The four uses:
//   decode rows     rows tokens  (A = k,  C = dy),  cols latents (B = q,  E = z),   row stats -> dk_dec
//   decode cols     rows latents (A = q,  C = z),   cols tokens  (B = k,  E = dy),  col stats -> dq_dec, dz
//   encode/synth.   rows tokens  (A = k,  C = v),   cols latents (B = q,  E = dO),  col stats -> dk, dv
//     token side
//   encode/synth.   rows latents (A = q,  C = dO),  cols tokens  (B = k,  E = v),   row stats -> dq
//     latent side
// (the synthesis has A = C = k0 on the token side and B = E = k0 on the latent
// side; its dk0 is scale acc1 + acc2).
// The decode's and the encode's token sides share the score S = k q^T and the
// product with q, so one "dual" launch serves both: a third row tile C2 = v
// and column tile E2 = dz give dPe = v dz^T, the weights Pd (row statistics)
// and Pe (column statistics) come from the same S, and
//     acc1 += (dSd + dSe) q  = dk / scale,     acc2 += Pe dz = dv.
//
// Per CTA (persistent, one per SM): NW softmax warpgroups, each with its own
// 128 rows, sharing every column tile, and one producer warpgroup:
//   warp 4NW          TMA: the item's row tiles (two slots) and a ring of
//                     column stages (B, E tiles and, with column statistics,
//                     the KT (lse, Delta) pairs by a bulk copy)
//   warps 4NW+1 ..    one MMA issuer per softmax warpgroup: S and dP of the
//                     next job are issued before the accumulating MMAs of the
//                     current one, so the tensor core runs ahead of the softmax
// TMEM per warpgroup: S and dP (KT columns each), acc1 and acc2 (max(D, 32)
// each), P and dS as packed 16-bit pairs (KT/2 each).  A job is KT = 32
// columns, or 64 where the job's products need one accumulator (AccForm):
// the latent sides of the encode and the synthesis (dq only), and the
// synthesis token side, whose two products are one gradient (dS is scaled
// before it is packed and both products add into acc1).  The dual launch
// defers each item's epilogue into the next item's first job.
// Every mbarrier wait is bounded as in the forward kernel (timeout recorded in
// the device status word, CTA-wide abort, bounded drain, TMEM freed).
#pragma once

#include "kernels_tc.cuh"

namespace flarepp {
namespace bwd_tc {

using tc::kQTile;

constexpr int kKT = 32;        // column tile rows of a job (one 32-column TMEM load per half)
constexpr int kKTWide = 64;    // passes with one accumulator: 64-column jobs

// How a job's accumulating products map to TMEM accumulators: one product
// (acc1 = dS B); two products into two accumulators (acc1 = dS B, acc2 =
// P E); two products into acc1 (acc1 = scale dS B + P E, dS scaled before it
// is packed: the synthesis token side, whose two products are one gradient).
enum AccForm { kAccOne = 0, kAccTwo = 1, kAccMerged = 2 };
constexpr int kNST = 4;        // column stages

// Tiles per row slot and per column stage, and row slots: the dual form holds
// three of each and one row slot (shared memory), the others two and two.
template <bool DUAL>
struct Shape {
    static constexpr int RT = DUAL ? 3 : 2;
    static constexpr int CT = DUAL ? 3 : 2;
    static constexpr int QS = DUAL ? 1 : 2;
};

enum Epilogue {
    kEpiPartials = 0,   // latent rows: acc1 (and acc2) -> fp32 partials [chunk][B*H][rows][D]
    kEpiTokDkDv = 2,    // token rows: dK = scale acc1, dV = acc2, in E   (decode + encode)
    kEpiTokDk0 = 3      // token rows: dK0 = scale acc1 + acc2, in E      (synthesis)
};

struct Params {
    int B, H;
    int row_count, col_count;   // rows and columns per (b, h)
    int col_tiles;              // ceil(col_count / KT)
    int row_groups;             // ceil(row_count / (NW 128))
    int chunks, chunk_tiles;    // column chunks per (b, h) and tiles per chunk
    int items;
    int row_tok, col_tok;       // rows / columns are token tensors
    int tok_heads_inner;        // token maps ordered (D, H, rows, B): [B,N,H,D] layout
    int a_shared, c_shared, b_shared, e_shared;   // [H,rows,D] tensors shared over the batch
    int c_same_a, e_same_b;     // C is A / E is B: one load serves both
    int has_acc2;
    int stats_per_col;          // lse, Delta per column (else per row); dual: per row
    const float2* stats;        // [B*H][stats_stride] (lse in log2 units, Delta)
    int64_t stats_stride;       // a multiple of KT (column statistics are bulk-copied per tile)
    const float2* stats2;       // dual: the column statistics of the second softmax
    int64_t stats2_stride;
    float scale_log2, scale;
    int epi;                    // Epilogue
    float* part1;
    float* part2;
    void* out1;                 // token outputs in E: dK (or dK0)
    void* out2;                 // dV
    int64_t tok_row, tok_h, tok_b;   // element strides of the token outputs
};

struct Item {
    int bh, h, b, row0, t_begin, t_end, chunk;
};

template <int NW>
__device__ __forceinline__ Item decode_item(const Params& p, int item) {
    Item it;
    const int g = item % p.row_groups;
    const int rest = item / p.row_groups;
    it.chunk = rest % p.chunks;
    it.bh = rest / p.chunks;
    it.h = it.bh % p.H;
    it.b = it.bh / p.H;
    it.row0 = g * NW * kQTile;
    it.t_begin = it.chunk * p.chunk_tiles;
    it.t_end = min(p.col_tiles, it.t_begin + p.chunk_tiles);
    return it;
}

template <int D, int NW, bool DUAL, int KT>
struct Smem {
    using SH = Shape<DUAL>;
    static constexpr int kRowTile = kQTile * D * 2;
    static constexpr int kColTile = KT * D * 2;
    static constexpr int kRow = 0;                                      // [QS][NW][A, C (, C2)]
    static constexpr int kCol = kRow + SH::QS * NW * SH::RT * kRowTile;  // [NST][B, E (, E2)]
    static constexpr int kStats = kCol + kNST * SH::CT * kColTile;      // [NST][KT] float2
    static constexpr int kBar = kStats + kNST * KT * 8;
    // row_full[QS], row_empty[QS], col_full[NST], col_empty[NST], sfull, sfree, pfull, pfree, drain [NW]
    static constexpr int kNumBars = 2 * SH::QS + 2 * kNST + 5 * NW;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kLaunchBytes = kBytes + 1024;
    // at least 116 KB so that a second CTA (which would block on TMEM) never shares the SM
    static constexpr int kSmemLaunch = kLaunchBytes > 118784 ? kLaunchBytes : 118784;
};

// TMEM columns of the plan: S, dP (, dP2) of KT columns, acc1 (, acc2 with
// kAccTwo) of max(D, 32), P and dS as packed pairs of KT/2, per warpgroup.
template <int D, int NW, bool DUAL, int KT, int ACC>
struct Tmem {
    static constexpr int OS = D < 32 ? 32 : D;
    static constexpr int kS = 0;
    static constexpr int kDP = NW * KT;
    static constexpr int kDP2 = 2 * NW * KT;                   // dual only
    static constexpr int kA1 = (DUAL ? 3 : 2) * NW * KT;
    static constexpr int kA2 = kA1 + NW * OS;                  // kAccTwo only
    static constexpr int kP = kA2 + (ACC == kAccTwo ? NW * OS : 0);
    static constexpr int kDS = kP + NW * (KT / 2);
    static constexpr int kTotal = kDS + NW * (KT / 2);
    static_assert(kTotal <= 512, "TMEM plan exceeds 512 columns");
    static_assert(ACC == kAccTwo || !DUAL, "the dual form accumulates two gradients");
};

// 16 consecutive TMEM columns of this thread's lane <- 16 registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(tc::smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(tc::smem_u32(bar))
                 : "memory");
}

template <typename E, int D, int NW, bool DUAL, int KT, int ACC>
__global__ void __launch_bounds__((NW + 1) * 128, 1)
bwd_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_c,
           const __grid_constant__ CUtensorMap map_c2, const __grid_constant__ CUtensorMap map_b,
           const __grid_constant__ CUtensorMap map_e, const __grid_constant__ CUtensorMap map_e2, const Params p) {
    static_assert(D == 16 || D == 32 || D == 64 || D == 128, "head dims 16, 32, 64, 128");
    static_assert(KT == 32 || KT == 64, "jobs of one or two 32-column halves");
    using SM = Smem<D, NW, DUAL, KT>;
    using TM = Tmem<D, NW, DUAL, KT, ACC>;
    using SH = Shape<DUAL>;
    using LY = tc::Layout<D, NW, KT>;
    constexpr int kHalves = KT / 32;
    constexpr int kQS = SH::QS;
    constexpr int kTmaWarp = 4 * NW;
    constexpr int kMmaWarp0 = 4 * NW + 1;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
    uint64_t* row_full = bars;
    uint64_t* row_empty = row_full + kQS;
    uint64_t* col_full = row_empty + kQS;
    uint64_t* col_empty = col_full + kNST;
    uint64_t* sfull = col_empty + kNST;
    uint64_t* sfree = sfull + NW;
    uint64_t* pfull = sfree + NW;
    uint64_t* pfree = pfull + NW;
    uint64_t* drain = pfree + NW;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kMisc + 4);
    const float2* sstats = reinterpret_cast<const float2*>(smem + SM::kStats);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kQS; ++i) { tc::mbar_init(&row_full[i], 1); tc::mbar_init(&row_empty[i], NW); }
        for (int i = 0; i < kNST; ++i) { tc::mbar_init(&col_full[i], 1); tc::mbar_init(&col_empty[i], NW); }
        for (int w = 0; w < NW; ++w) {
            tc::mbar_init(&sfull[w], 1);
            tc::mbar_init(&sfree[w], 4);
            tc::mbar_init(&pfull[w], 4);
            tc::mbar_init(&pfree[w], 1);
            tc::mbar_init(&drain[w], 1);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kTmaWarp && lane == 0) {
        tc::prefetch_tensormap(&map_a);
        tc::prefetch_tensormap(&map_c);
        tc::prefetch_tensormap(&map_b);
        tc::prefetch_tensormap(&map_e);
        if (DUAL) {
            tc::prefetch_tensormap(&map_c2);
            tc::prefetch_tensormap(&map_e2);
        }
    }
    if (warp == kMmaWarp0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(tc::smem_u32(tmem_slot)), "r"(tc::kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();
    pdl_launch_dependents();
    // Registers: with two softmax warpgroups the launch gives 168 per thread; the
    // producer warpgroup gives back down to 56 and the softmax warpgroups rise to
    // 224 (2 x 128 x 224 + 128 x 56 = 384 x 168).  The build refuses a library whose
    // launch allocation for this kernel is not exactly 168, since a larger `inc`
    // than the pool holds would wait forever.
    static_assert(NW != 2 || tc::Regs<2>::kSoftmax == 224, "register split of the backward kernel");

    if (warp >= 4 * NW) {
      if constexpr (NW == 2) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(tc::kProducerRegs));
      if (warp == kTmaWarp) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t ic = 0, g = 0;
            int col_last[kNST], row_last[kQS];
            for (int i = 0; i < kNST; ++i) col_last[i] = -1;
            for (int i = 0; i < kQS; ++i) row_last[i] = -1;
            const bool col_stats = DUAL || p.stats_per_col;
            const uint32_t row_bytes = NW * ((p.c_same_a ? 1 : 2) + (DUAL ? 1 : 0)) * SM::kRowTile;
            const uint32_t col_bytes =
                ((p.e_same_b ? 1 : 2) + (DUAL ? 1 : 0)) * SM::kColTile + (col_stats ? KT * 8 : 0);
            const float2* cstats = DUAL ? p.stats2 : p.stats;
            const int64_t cstride = DUAL ? p.stats2_stride : p.stats_stride;
            bool ok = true;
            // coordinates of a tile of `rows` starting at row r of (b, h): token maps may be
            // ordered (D, H, rows, B); latent maps are always (D, rows, H, B)
            auto load = [&](void* dst, const CUtensorMap* map, uint64_t* bar, bool tok, int cb, int r, int h, int b) {
                if (tok && p.tok_heads_inner) tc::tma_load_4d(dst, map, bar, cb * 64, h, r, b);
                else tc::tma_load_4d(dst, map, bar, cb * 64, r, h, b);
            };
            for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
                const Item it = decode_item<NW>(p, item);
                const int slot = ic % kQS;
                ok = tc::mbar_wait(&row_empty[slot], ((ic / kQS) & 1) ^ 1, abort_flag);
                if (!ok) break;
                tc::mbar_expect_tx(&row_full[slot], row_bytes);
                uint8_t* rdst = smem + SM::kRow + slot * NW * SH::RT * SM::kRowTile;
                for (int w = 0; w < NW; ++w) {
                    const int r = it.row0 + w * kQTile;
                    uint8_t* wdst = rdst + w * SH::RT * SM::kRowTile;
#pragma unroll
                    for (int cb = 0; cb < LY::kBlocks; ++cb) {
                        load(wdst + cb * LY::kQBlockBytes, &map_a, &row_full[slot], p.row_tok, cb, r, it.h,
                             p.a_shared ? 0 : it.b);
                        if (!p.c_same_a)
                            load(wdst + SM::kRowTile + cb * LY::kQBlockBytes, &map_c, &row_full[slot], p.row_tok,
                                 cb, r, it.h, p.c_shared ? 0 : it.b);
                        if (DUAL)   // C2: the second output-gradient operand (same batch as the tokens)
                            load(wdst + 2 * SM::kRowTile + cb * LY::kQBlockBytes, &map_c2, &row_full[slot],
                                 p.row_tok, cb, r, it.h, it.b);
                    }
                }
                row_last[slot] = (ic / kQS) & 1;
                ++ic;
                for (int t = it.t_begin; t < it.t_end; ++t) {
                    const int st = g % kNST;
                    ok = tc::mbar_wait(&col_empty[st], ((g / kNST) & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    tc::mbar_expect_tx(&col_full[st], col_bytes);
                    uint8_t* cdst = smem + SM::kCol + st * SH::CT * SM::kColTile;
#pragma unroll
                    for (int cb = 0; cb < LY::kBlocks; ++cb) {
                        load(cdst + cb * LY::kKVBlockBytes, &map_b, &col_full[st], p.col_tok, cb, t * KT, it.h,
                             p.b_shared ? 0 : it.b);
                        if (!p.e_same_b)
                            load(cdst + SM::kColTile + cb * LY::kKVBlockBytes, &map_e, &col_full[st], p.col_tok, cb,
                                 t * KT, it.h, p.e_shared ? 0 : it.b);
                        if (DUAL)   // E2: the second output gradient's column tile (per batch)
                            load(cdst + 2 * SM::kColTile + cb * LY::kKVBlockBytes, &map_e2, &col_full[st], p.col_tok,
                                 cb, t * KT, it.h, it.b);
                    }
                    if (col_stats)
                        bulk_load(smem + SM::kStats + st * KT * 8, cstats + it.bh * cstride + t * KT, KT * 8,
                                  &col_full[st]);
                    col_last[st] = (g / kNST) & 1;
                    ++g;
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA exits (bounded)
                const unsigned long long t0 = tc::globaltimer_ns();
                for (int s = 0; s < kNST; ++s)
                    while (col_last[s] >= 0 && !tc::mbar_try_wait(&col_full[s], col_last[s]) &&
                           tc::globaltimer_ns() - t0 < 100000000ull) {
                    }
                for (int s = 0; s < kQS; ++s)
                    while (row_last[s] >= 0 && !tc::mbar_try_wait(&row_full[s], row_last[s]) &&
                           tc::globaltimer_ns() - t0 < 100000000ull) {
                    }
            }
        }
      } else {
        // ---------------------------------------------------------- MMA issuers
        if (lane == 0 && warp < kMmaWarp0 + NW) {
            const int w = warp - kMmaWarp0;
            constexpr uint32_t idesc_s = tc::make_idesc(kQTile, KT, false, tc::Elem<E>::kFmt);  // [128 x KT]
            constexpr uint32_t idesc_a = tc::make_idesc(kQTile, D, true, tc::Elem<E>::kFmt);     // [128 x D], B MN-major
            // The job stream of this CTA: every column tile of every item, in order.
            struct Job {
                int item, t;
                Item info;
                uint32_t ic, g;
                bool valid;
            };
            auto first_job = [&](Job& j) {
                j.item = blockIdx.x;
                j.ic = 0;
                j.g = 0;
                j.valid = j.item < p.items;
                if (j.valid) {
                    j.info = decode_item<NW>(p, j.item);
                    j.t = j.info.t_begin;
                }
            };
            auto next_job = [&](Job& j) {
                ++j.g;
                if (++j.t < j.info.t_end) return;
                ++j.ic;
                j.item += gridDim.x;
                j.valid = j.item < p.items;
                if (j.valid) {
                    j.info = decode_item<NW>(p, j.item);
                    j.t = j.info.t_begin;
                }
            };
            bool ok = true;
            uint32_t s_issued = 0, a_issued = 0;
            auto issue_s = [&](const Job& j) -> bool {
                const int slot = j.ic % kQS;
                if (j.t == j.info.t_begin && !tc::mbar_wait(&row_full[slot], (j.ic / kQS) & 1, abort_flag))
                    return false;
                const int st = j.g % kNST;
                if (!tc::mbar_wait(&col_full[st], (j.g / kNST) & 1, abort_flag)) return false;
                if (!tc::mbar_wait(&sfree[w], (s_issued & 1) ^ 1, abort_flag)) return false;
                tc::tc_fence_after();
                const uint8_t* rbase = smem + SM::kRow + (slot * NW + w) * SH::RT * SM::kRowTile;
                const uint32_t aaddr = tc::smem_u32(rbase);
                const uint32_t caddr = tc::smem_u32(p.c_same_a ? rbase : rbase + SM::kRowTile);
                const uint8_t* cbase = smem + SM::kCol + st * SH::CT * SM::kColTile;
                const uint32_t baddr = tc::smem_u32(cbase);
                const uint32_t eaddr = tc::smem_u32(p.e_same_b ? cbase : cbase + SM::kColTile);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = tc::smem_desc(aaddr + LY::kstep(kk, LY::kQBlockBytes), 16, LY::kSbo, LY::kType);
                    const uint64_t bd = tc::smem_desc(baddr + LY::kstep(kk, LY::kKVBlockBytes), 16, LY::kSbo, LY::kType);
                    tc::umma_f16(tmem + TM::kS + w * KT, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t cd = tc::smem_desc(caddr + LY::kstep(kk, LY::kQBlockBytes), 16, LY::kSbo, LY::kType);
                    const uint64_t ed = tc::smem_desc(eaddr + LY::kstep(kk, LY::kKVBlockBytes), 16, LY::kSbo, LY::kType);
                    tc::umma_f16(tmem + TM::kDP + w * KT, cd, ed, idesc_s, kk > 0 ? 1u : 0u);
                }
                if constexpr (DUAL) {
                    const uint32_t c2addr = tc::smem_u32(rbase + 2 * SM::kRowTile);
                    const uint32_t e2addr = tc::smem_u32(cbase + 2 * SM::kColTile);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t cd =
                            tc::smem_desc(c2addr + LY::kstep(kk, LY::kQBlockBytes), 16, LY::kSbo, LY::kType);
                        const uint64_t ed =
                            tc::smem_desc(e2addr + LY::kstep(kk, LY::kKVBlockBytes), 16, LY::kSbo, LY::kType);
                        tc::umma_f16(tmem + TM::kDP2 + w * KT, cd, ed, idesc_s, kk > 0 ? 1u : 0u);
                    }
                }
                tc::umma_commit(&sfull[w]);
                ++s_issued;
                // the last score MMAs of the item release this warpgroup's share of the row slot
                if (j.t + 1 >= j.info.t_end) tc::umma_commit(&row_empty[slot]);
                return true;
            };
            auto issue_acc = [&](const Job& j) -> bool {
                if (!tc::mbar_wait(&pfull[w], a_issued & 1, abort_flag)) return false;
                tc::tc_fence_after();
                const int st = j.g % kNST;
                const uint8_t* cbase = smem + SM::kCol + st * SH::CT * SM::kColTile;
                const uint32_t baddr = tc::smem_u32(cbase);
                // acc2's B operand: E, or E2 in the dual form (acc2 = Pe E2)
                const uint32_t eaddr = tc::smem_u32(DUAL ? cbase + 2 * SM::kColTile
                                                         : (p.e_same_b ? cbase : cbase + SM::kColTile));
                const bool first = j.t == j.info.t_begin;
#pragma unroll
                for (int kk = 0; kk < KT / 16; ++kk) {
                    // A = dS (or P) in TMEM: 16 columns of the tile = 8 packed TMEM columns per step;
                    // B = the column tile [KT x D], D contiguous: MN-major, 16 rows per step
                    const uint64_t bd = tc::smem_desc(baddr + kk * 16 * LY::kRowBytes, LY::kKVBlockBytes, LY::kSbo,
                                                      LY::kType);
                    tc::umma_f16_tmem_a(tmem + TM::kA1 + w * TM::OS, tmem + TM::kDS + w * (KT / 2) + kk * 8, bd,
                                        idesc_a, (first && kk == 0) ? 0u : 1u);
                }
                if (ACC == kAccMerged || (ACC == kAccTwo && p.has_acc2)) {
                    // the second product: into acc2, or added to acc1 (kAccMerged)
                    const uint32_t acc = ACC == kAccMerged ? TM::kA1 : TM::kA2;
#pragma unroll
                    for (int kk = 0; kk < KT / 16; ++kk) {
                        const uint64_t ed = tc::smem_desc(eaddr + kk * 16 * LY::kRowBytes, LY::kKVBlockBytes,
                                                          LY::kSbo, LY::kType);
                        tc::umma_f16_tmem_a(tmem + acc + w * TM::OS, tmem + TM::kP + w * (KT / 2) + kk * 8, ed,
                                            idesc_a, (ACC == kAccTwo && first && kk == 0) ? 0u : 1u);
                    }
                }
                tc::umma_commit(&pfree[w]);
                tc::umma_commit(&col_empty[st]);
                ++a_issued;
                return true;
            };
            Job sj, aj;
            first_job(sj);
            first_job(aj);
            if (sj.valid) {
                ok = issue_s(sj);
                next_job(sj);
            }
            while (aj.valid && ok) {
                if (sj.valid) {
                    ok = issue_s(sj);
                    if (!ok) break;
                    next_job(sj);
                }
                ok = issue_acc(aj);
                next_job(aj);
            }
            // drain: every issued MMA completes before TMEM is released; if that
            // runs out, report it (the outputs are then undefined)
            tc::umma_commit(&drain[w]);
            const unsigned long long t0 = tc::globaltimer_ns();
            bool drained = false;
            while (!(drained = tc::mbar_try_wait(&drain[w], 0)) && tc::globaltimer_ns() - t0 < tc::kWaitLimitNs) {
            }
            if (!drained) {
                *abort_flag = 1;
                record_status(tc::kStatusTimeout);
            }
        }
      }
    } else {
        if constexpr (NW == 2) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(tc::Regs<2>::kSoftmax));
        // ---------------------------------------------------------- softmax warpgroups
        const int wg = warp >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + TM::kS + wg * KT;
        const uint32_t tDP = tmem + lane_base + TM::kDP + wg * KT;
        const uint32_t tDP2 = tmem + lane_base + TM::kDP2 + wg * KT;
        const uint32_t tA1 = tmem + lane_base + TM::kA1 + wg * TM::OS;
        const uint32_t tA2 = tmem + lane_base + TM::kA2 + wg * TM::OS;
        const uint32_t tP = tmem + lane_base + TM::kP + wg * (KT / 2);
        const uint32_t tDS = tmem + lane_base + TM::kDS + wg * (KT / 2);
        const float sl2 = p.scale_log2;
        uint32_t sfull_waits = 0, pfree_waits = 0, jobs_done = 0, g = 0;
        bool ok = true;
        // An item's accumulators -> its outputs (every accumulating MMA of the
        // item has completed).  The fused token side (DUAL: items of 16 jobs)
        // defers it into the next item's first job: the item's last
        // accumulation finishes in the shadow of the next exponentials, and
        // the accumulators are read after that job's P and dS stores, before
        // its pfull releases the MMA that resets them.  The other forms (items
        // of hundreds of jobs, or a single softmax per job) ran faster with it
        // at the end of the item.
        auto epilogue = [&](const Item& it, int r, bool rvalid) {
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                constexpr int CW = D < 32 ? D : 32;        // valid columns of a 32-column load
                uint32_t a1[32], a2[32];
                tc::tmem_ld32(tA1 + c0, a1);
                if (ACC == kAccTwo && p.has_acc2) tc::tmem_ld32(tA2 + c0, a2);
                tc::tmem_wait_ld();
                if (!rvalid) continue;
                if (p.epi == kEpiPartials) {
                    const int64_t ridx = ((int64_t)it.chunk * p.B * p.H + it.bh) * p.row_count + r;
                    float4* d1 = reinterpret_cast<float4*>(p.part1 + ridx * D + c0);
#pragma unroll
                    for (int i = 0; i < CW / 4; ++i)
                        d1[i] = make_float4(__uint_as_float(a1[4 * i]), __uint_as_float(a1[4 * i + 1]),
                                            __uint_as_float(a1[4 * i + 2]), __uint_as_float(a1[4 * i + 3]));
                    if (ACC == kAccTwo && p.has_acc2) {
                        float4* d2 = reinterpret_cast<float4*>(p.part2 + ridx * D + c0);
#pragma unroll
                        for (int i = 0; i < CW / 4; ++i)
                            d2[i] = make_float4(__uint_as_float(a2[4 * i]), __uint_as_float(a2[4 * i + 1]),
                                                __uint_as_float(a2[4 * i + 2]), __uint_as_float(a2[4 * i + 3]));
                    }
                } else if constexpr (ACC != kAccOne) {
                    const int64_t off = (int64_t)it.b * p.tok_b + (int64_t)it.h * p.tok_h + (int64_t)r * p.tok_row + c0;
                    float v1[CW];
                    if (p.epi == kEpiTokDkDv) {
#pragma unroll
                        for (int i = 0; i < CW; ++i) v1[i] = p.scale * __uint_as_float(a1[i]);
                        float v2[CW];
#pragma unroll
                        for (int i = 0; i < CW; ++i) v2[i] = __uint_as_float(a2[i]);
                        store_row<E, CW>(static_cast<E*>(p.out2) + off, v2);
                    } else if constexpr (ACC == kAccMerged) {
#pragma unroll
                        for (int i = 0; i < CW; ++i) v1[i] = __uint_as_float(a1[i]);      // scale dS B + P E
                    } else {
#pragma unroll
                        for (int i = 0; i < CW; ++i)
                            v1[i] = fmaf(p.scale, __uint_as_float(a1[i]), __uint_as_float(a2[i]));
                    }
                    store_row<E, CW>(static_cast<E*>(p.out1) + off, v1);
                }
            }
        };
        bool pend = false;
        Item pend_it{};
        int pend_r = 0;
        bool pend_rvalid = false;
        for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
            const Item it = decode_item<NW>(p, item);
            const int r = it.row0 + wg * kQTile + row;
            const bool rvalid = r < p.row_count;
            const bool warp_rows_valid = it.row0 + wg * kQTile + wq * 32 + 31 < p.row_count;
            float lse_r = 0.f, del_r = 0.f;
            if ((DUAL || !p.stats_per_col) && rvalid) {
                const float2 sv = p.stats[it.bh * p.stats_stride + r];
                lse_r = sv.x;
                del_r = sv.y;
            }
            for (int t = it.t_begin; t < it.t_end; ++t, ++g) {
                if (!tc::mbar_wait(&sfull[wg], sfull_waits & 1, abort_flag)) { ok = false; break; }
                ++sfull_waits;
                tc::tc_fence_after();
                uint32_t sr[kHalves][32], dr[kHalves][32], dr2[DUAL ? kHalves : 1][DUAL ? 32 : 1];
#pragma unroll
                for (int h = 0; h < kHalves; ++h) {
                    tc::tmem_ld32(tS + 32 * h, sr[h]);
                    tc::tmem_ld32(tDP + 32 * h, dr[h]);
                    if constexpr (DUAL) tc::tmem_ld32(tDP2 + 32 * h, dr2[h]);
                }
                tc::tmem_wait_ld();
                tc::tc_fence_before();
                __syncwarp();
                tc::mbar_arrive_if(&sfree[wg], lane == 0);

                const int st = g % kNST;
                if (DUAL || p.stats_per_col) {
                    // the stage's statistics: acquire the TMA writes (the phase has completed)
                    if (!tc::mbar_wait(&col_full[st], (g / kNST) & 1, abort_flag)) { ok = false; break; }
                }
#pragma unroll
                for (int h = 0; h < kHalves; ++h) {
                    const float2* cs = sstats + st * KT + 32 * h;
                    const int valid = p.col_count - t * KT - 32 * h;     // columns of this half that exist
                    uint32_t pk[16], dk[16];
                    if (__builtin_expect(valid >= 32 && warp_rows_valid, 1)) {
                        // every row of the warp and every column of the tile exists (warp-uniform):
                        // no masking, column pairs in packed fp32 arithmetic
                        const float2 sl2v = make_float2(sl2, sl2);
                        const float2 nlr = make_float2(-lse_r, -lse_r), ndr = make_float2(-del_r, -del_r);
                        const float4* cs4 = reinterpret_cast<const float4*>(cs);
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float2 s2 = make_float2(__uint_as_float(sr[h][2 * j]), __uint_as_float(sr[h][2 * j + 1]));
                            const float2 d2 = make_float2(__uint_as_float(dr[h][2 * j]), __uint_as_float(dr[h][2 * j + 1]));
                            float2 pw, ds;
                            if constexpr (DUAL) {
                                const float4 sv = cs4[j];                    // (lse, Delta) of columns 2j, 2j+1
                                const float2 xd = __ffma2_rn(s2, sl2v, nlr);
                                const float2 xe = __ffma2_rn(s2, sl2v, make_float2(-sv.x, -sv.z));
                                const float2 pd = make_float2(ex2_mufu(xd.x), ex2_mufu(xd.y));
                                pw = make_float2(ex2_mufu(xe.x), ex2_mufu(xe.y));
                                const float2 e2 = make_float2(__uint_as_float(dr2[h][2 * j]), __uint_as_float(dr2[h][2 * j + 1]));
                                const float2 ge = __fmul2_rn(pw, __fadd2_rn(e2, make_float2(-sv.y, -sv.w)));
                                ds = __ffma2_rn(pd, __fadd2_rn(d2, ndr), ge);
                            } else {
                                float2 nl = nlr, nd = ndr;
                                if (p.stats_per_col) {
                                    const float4 sv = cs4[j];
                                    nl = make_float2(-sv.x, -sv.z);
                                    nd = make_float2(-sv.y, -sv.w);
                                }
                                const float2 x = __ffma2_rn(s2, sl2v, nl);
                                pw = make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
                                ds = __fmul2_rn(pw, __fadd2_rn(d2, nd));
                                if constexpr (ACC == kAccMerged) ds = __fmul2_rn(ds, make_float2(p.scale, p.scale));
                            }
                            pk[j] = pack2<E>(pw.x, pw.y);
                            dk[j] = pack2<E>(ds.x, ds.y);
                        }
                    } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float pv[2], dv[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int c = 2 * j + e;
                            const bool on = rvalid && c < valid;
                            const float sc = __uint_as_float(sr[h][c]);
                            if constexpr (DUAL) {
                                // Pd from the row statistics (first softmax), Pe from the column
                                // statistics (second); dS = dSd + dSe, the weights stored are Pe
                                const float2 sv = cs[c];
                                const float pd = on ? ex2_mufu(fmaf(sc, sl2, -lse_r)) : 0.f;
                                const float pe = on ? ex2_mufu(fmaf(sc, sl2, -sv.x)) : 0.f;
                                pv[e] = pe;
                                dv[e] = on ? fmaf(pd, __uint_as_float(dr[h][c]) - del_r, pe * (__uint_as_float(dr2[h][c]) - sv.y))
                                           : 0.f;
                            } else {
                                float lse = lse_r, del = del_r;
                                if (p.stats_per_col) {
                                    const float2 sv = cs[c];
                                    lse = sv.x;
                                    del = sv.y;
                                }
                                const float x = fmaf(sc, sl2, -lse);
                                const float pw = on ? ex2_mufu(x) : 0.f;
                                pv[e] = pw;
                                dv[e] = on ? pw * (__uint_as_float(dr[h][c]) - del) : 0.f;
                                if constexpr (ACC == kAccMerged) dv[e] *= p.scale;
                            }
                        }
                        pk[j] = pack2<E>(pv[0], pv[1]);
                        dk[j] = pack2<E>(dv[0], dv[1]);
                    }
                    }
                    if (h == 0) {
                        // the previous job's accumulating MMAs must be done before P and dS are overwritten
                        while (pfree_waits < jobs_done) {
                            if (!tc::mbar_wait(&pfree[wg], pfree_waits & 1, abort_flag)) { ok = false; break; }
                            ++pfree_waits;
                        }
                        if (!ok) break;
                        tc::tc_fence_after();
                    }
                    tmem_st16(tP + 16 * h, pk);
                    tmem_st16(tDS + 16 * h, dk);
                }
                if (!ok) break;
                if constexpr (DUAL) {
                    if (pend) {
                        epilogue(pend_it, pend_r, pend_rvalid);
                        pend = false;
                    }
                }
                tc::tmem_wait_st();
                tc::tc_fence_before();
                __syncwarp();
                tc::mbar_arrive_if(&pfull[wg], lane == 0);
                ++jobs_done;
            }
            if (!ok) break;

            // ---------------- end of the item
            if constexpr (DUAL) {
                pend = true;         // its epilogue waits for the next item's first job
                pend_it = it;
                pend_r = r;
                pend_rvalid = rvalid;
            } else {
                while (pfree_waits < jobs_done) {
                    if (!tc::mbar_wait(&pfree[wg], pfree_waits & 1, abort_flag)) { ok = false; break; }
                    ++pfree_waits;
                }
                if (!ok) break;
                tc::tc_fence_after();
                epilogue(it, r, rvalid);
                // the accumulators are read before the next item's first job is released to the MMA
                tc::tc_fence_before();
            }
        }
        if (ok && pend) {
            // the last item's epilogue, once its last accumulating MMA has completed
            while (pfree_waits < jobs_done) {
                if (!tc::mbar_wait(&pfree[wg], pfree_waits & 1, abort_flag)) { ok = false; break; }
                ++pfree_waits;
            }
            if (ok) {
                tc::tc_fence_after();
                epilogue(pend_it, pend_r, pend_rvalid);
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp0) {
        tc::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tc::kTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------ host side

// One tensor operand of the kernel: a latent tensor ([H,M,D] shared over the
// batch, or [B,H,M,D]) or a token tensor (token layout strides).
struct Operand {
    const void* ptr;
    bool tok;
    bool shared;
};

struct Launch {
    int B, H, N, M, D;
    tc::RowStrides tok;
    Operand a, c, b, e;
    bool dual;                 // the fused decode + encode token side (c2, e2, stats2 used)
    Operand c2, e2;
    const float2* stats2;
    int64_t stats2_stride;
    bool rows_tok;             // rows are tokens (N rows), else latents (M rows)
    bool has_acc2, stats_per_col;
    const float2* stats;
    int64_t stats_stride;
    float scale_log2, scale;
    int epi;
    int chunk_len;             // latent rows: tokens per column chunk, a multiple of kKTWide (0 = planned)
    float *part1, *part2;
    void *out1, *out2;
};

// Warpgroups per CTA: two for D <= 64 (TMEM: 2 x (3 KT + 2 max(D, 32)) <= 512),
// one for D = 128.
constexpr int nw_for(int D) { return D == 128 ? 1 : 2; }

// Tokens per column chunk of the latent-row passes: the forward split pass's
// cost model (waves x (fixed work + jobs per item)) over 64-token tiles, or
// `force` chunks.  A multiple of kKTWide, so that every latent-row pass,
// whatever its job width, splits the tokens at the same places and writes
// the same partial slots.
inline int plan_chunk_len(int B, int H, int M, int N, int D, int force) {
    const int NW = nw_for(D);
    const int64_t units = (int64_t)B * H * ((M + NW * kQTile - 1) / (NW * kQTile));
    const int64_t tiles = (N + kKTWide - 1) / kKTWide;
    const int64_t chunks = force > 0 ? std::min<int64_t>(force, tiles) : tc::choose_chunks(units, tiles, kNumSMs, 1);
    const int64_t per = (tiles + chunks - 1) / chunks;
    return (int)(per * kKTWide);
}

// Column chunks of a latent-row pass with `chunk_len` tokens per chunk.
inline int chunks_of(int N, int chunk_len) { return (int)(((int64_t)N + chunk_len - 1) / chunk_len); }

template <typename E, int D, bool DUAL, int KT, int ACC>
int launch_bwd_kt(const Launch& L, cudaStream_t st) {
    constexpr int NW = nw_for(D);
    using SM = Smem<D, NW, DUAL, KT>;
    static_assert(SM::kLaunchBytes <= 232448, "shared memory plan exceeds 227 KB");
    const CUtensorMapDataType ty = tc::Elem<E>::kMapType;
    const tc::RowStrides lat = tc::contiguous_rows(L.M, L.H, D);
    auto map = [&](CUtensorMap* m, const Operand& o, int box) {
        if (o.tok) return tc::make_map(m, ty, o.ptr, L.N, L.H, L.B, D, L.tok, box);
        return tc::make_map(m, ty, o.ptr, L.M, L.H, o.shared ? 1 : L.B, D, lat, box);
    };
    CUtensorMap ma, mc, mb, me, mc2, me2;
    if (!map(&ma, L.a, kQTile) || !map(&mc, L.c, kQTile) || !map(&mb, L.b, KT) || !map(&me, L.e, KT)) return 3;
    if (DUAL) {
        if (!map(&mc2, L.c2, kQTile) || !map(&me2, L.e2, KT)) return 3;
    } else {
        mc2 = mc;
        me2 = me;
    }
    Params p{};
    p.B = L.B; p.H = L.H;
    p.row_count = L.rows_tok ? L.N : L.M;
    p.col_count = L.rows_tok ? L.M : L.N;
    p.col_tiles = (p.col_count + KT - 1) / KT;
    p.row_groups = (p.row_count + NW * kQTile - 1) / (NW * kQTile);
    if (L.rows_tok) {
        p.chunk_tiles = p.col_tiles;          // an item holds all the latents
    } else {
        const int len = L.chunk_len > 0 ? L.chunk_len : plan_chunk_len(L.B, L.H, L.M, L.N, D, 0);
        if (len % kKTWide != 0) return 2;
        p.chunk_tiles = len / KT;
    }
    p.chunks = (p.col_tiles + p.chunk_tiles - 1) / p.chunk_tiles;
    p.items = L.B * L.H * p.chunks * p.row_groups;
    p.row_tok = L.rows_tok ? 1 : 0;
    p.col_tok = L.rows_tok ? 0 : 1;
    p.tok_heads_inner = L.tok.h < L.tok.row ? 1 : 0;
    p.a_shared = L.a.shared; p.c_shared = L.c.shared; p.b_shared = L.b.shared; p.e_shared = L.e.shared;
    p.c_same_a = L.c.ptr == L.a.ptr ? 1 : 0;
    p.e_same_b = L.e.ptr == L.b.ptr ? 1 : 0;
    p.has_acc2 = L.has_acc2 ? 1 : 0;
    p.stats_per_col = L.stats_per_col ? 1 : 0;
    p.stats = L.stats;
    p.stats_stride = L.stats_stride;
    p.stats2 = L.stats2;
    p.stats2_stride = L.stats2_stride;
    p.scale_log2 = L.scale_log2;
    p.scale = L.scale;
    p.epi = L.epi;
    p.part1 = L.part1; p.part2 = L.part2;
    p.out1 = L.out1; p.out2 = L.out2;
    p.tok_row = L.tok.row; p.tok_h = L.tok.h; p.tok_b = L.tok.b;
    if (ACC == kAccOne && L.has_acc2) return 2;
    if (ACC == kAccMerged && (!L.has_acc2 || L.epi != kEpiTokDk0)) return 2;
    auto kern = bwd_kernel<E, D, NW, DUAL, KT, ACC>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kSmemLaunch) != cudaSuccess)
        return 3;
    const int grid = p.items < tc::sm_count() ? p.items : tc::sm_count();
    return tc::launch_pdl(kern, dim3(grid), dim3((NW + 1) * 128), SM::kSmemLaunch, st, ma, mc, mc2, mb, me, me2,
                          p) == cudaSuccess
               ? 0
               : 3;
}

// Job width: with two warpgroups, a pass with one accumulator takes
// 64-column jobs (TMEM: 2 x (64 S + 64 dP + 64 acc1 + 32 P + 32 dS) = 512;
// the per-job synchronisation is spread over twice the columns): the latent
// sides of the encode and the synthesis (one product, row statistics) and the
// synthesis token side (two products merged into acc1).  The decode's latent
// side and the fused token side keep two accumulators and 32-column jobs.
template <typename E, int D, bool DUAL>
int launch_bwd(const Launch& L, cudaStream_t st) {
    if constexpr (!DUAL && nw_for(D) == 2) {
        if (!L.rows_tok && !L.has_acc2 && !L.stats_per_col)
            return launch_bwd_kt<E, D, false, kKTWide, kAccOne>(L, st);
        if (L.rows_tok && L.has_acc2 && L.epi == kEpiTokDk0)
            return launch_bwd_kt<E, D, false, kKTWide, kAccMerged>(L, st);
    }
    return launch_bwd_kt<E, D, DUAL, kKT, kAccTwo>(L, st);
}

template <typename E, int D>
int launch_bwd_dual(const Launch& L, cudaStream_t st) {
    return L.dual ? launch_bwd<E, D, true>(L, st) : launch_bwd<E, D, false>(L, st);
}

template <typename E>
int launch_bwd_d(const Launch& L, cudaStream_t st) {
    switch (L.D) {
        case 16: return launch_bwd_dual<E, 16>(L, st);
        case 32: return launch_bwd_dual<E, 32>(L, st);
        case 64: return launch_bwd_dual<E, 64>(L, st);
        case 128: return launch_bwd_dual<E, 128>(L, st);
        default: return 2;
    }
}

}  // namespace bwd_tc
}  // namespace flarepp
