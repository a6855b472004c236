// tcgen05 (5th-generation tensor core) kernels of the FLARE++ mixer, 16-bit
// I/O (bf16 or fp16; the element type E is a template parameter throughout).
//
// One warp-specialised attention kernel serves all three SDPA calls of the
// FLARE++ block (FLARE.py README, "FLARE++" code block):
//   * split mode  -- synthesis q_dyn = SDPA(q0, k0, k0) and encode
//                    z = SDPA(q, k, v): the query rows are the M latents, the
//                    key/value rows are one chunk of the N tokens, and the
//                    output is the online-softmax triple (row max, row sum,
//                    unnormalised weighted sum) of every latent over the chunk,
//                    merged across chunks by merge_partials (log-sum-exp
//                    combine; physicsnemo issue #2024, section 2);
//   * decode mode -- y = SDPA(k, q, z): the query rows are tokens, the
//                    key/value rows are the M latents of q and z, and the
//                    output is the normalised y row in E.
//
// Per CTA (persistent, one per SM): NW query-row tiles of 128 rows, each served
// by CS softmax warpgroups (column shares: CS = 2 in the split passes at
// D = 64, else 1), and one producer warpgroup, (NW CS + 1) x 128 threads.
//   warps 0 .. 4NW CS-1  softmax warpgroup g = warp / 4 serves row tile g / CS
//                        and column share g % CS (TMEM lanes 32 (warp % 4) .. +31)
//   warp  4NW CS         TMA producer: query tiles and a ring of key/value tiles
//                        of KT rows
//   next NW warps        one MMA issuer per row tile w:
//                        S_w = Q_w K^T and O_w += P_w V, into TMEM
// TMEM columns: S_w at KT w, O_w at NW KT + OS w (OS = max(D, 32)), P_w (KT
// 16-bit values = KT/2 columns) after them; NW (KT + OS + KT/2) <= 512.
// Each softmax thread owns one query row (with CS = 2, KT/2 of its score
// columns, the matching P columns and D/2 of its O columns; the two warps on a
// lane quarter swap their half-row maxima through shared memory every job and
// their half-row sums at the end of an item): it reads its scores from TMEM,
// takes exponentials base 2, writes the weights P back to TMEM in E (the value
// MMA reads its A operand from TMEM), and rescales its O columns in TMEM only
// when its running max grows by more than 2^8 (the final normalisation uses the
// same stale max, so the result is exact up to rounding).  Each MMA warp
// issues its row tile's next score MMA as soon as the softmax has read the
// previous scores, before that job's value MMA, so the tensor core works ahead
// of the softmax; the row tiles run independently.
// Query tiles and key/value tiles are shared in one of two ways:
//   * shared key/value tiles (decode, and split with one 128-latent group per
//     row tile): each row tile has its own query tile and every row tile
//     consumes every key/value tile of the item;
//   * interleaved (split with M <= 128): the row tiles share one query tile and
//     take the item's key/value tiles round-robin, each writing its own
//     partial triple.
// The launch gives every thread R0 = 65536 / threads registers; the producer
// warpgroup gives back down to 56 and the softmax warpgroups take the rest
// (setmaxnreg), never more than the launch holds.  The build checks ptxas's
// launch allocation for each configuration.
//
// Every wait on an mbarrier is bounded (about 2 s of %globaltimer); on expiry
// the kernel records FLAREPP_ERR_TIMEOUT in the device status word, raises a
// CTA-wide abort flag that every other wait checks, drains its outstanding
// tensor-core work (bounded), frees its TMEM and returns.
#pragma once

#include <cuda.h>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "kernels_simt.cuh"

namespace flarepp {
namespace tc {

constexpr int kQTile = 128;          // query rows per tile (the tcgen05.mma M)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr int kStatusTimeout = 5;    // FLAREPP_ERR_TIMEOUT
constexpr int kProducerRegs = 56;    // producer warpgroup after setmaxnreg.dec

// Threads, launch registers and the register split of a configuration with NW
// softmax warpgroups and one producer warpgroup: the producer gives back down
// to kProducer and the softmax warpgroups take the rest (a producer share of
// 32 with four softmax warpgroups measured slower: its code spills).
template <int NW>
struct Regs {
    static constexpr int kThreads = (NW + 1) * 128;
    static constexpr int kLaunch = (65536 / kThreads) / 8 * 8;           // 168 (NW=2), 128 (NW=3), 96 (NW=4)
    static constexpr int kProducer = kProducerRegs;
    static constexpr int kSoftmax = ((kThreads * kLaunch - 128 * kProducer) / (NW * 128)) / 8 * 8;
    static_assert(NW * 128 * kSoftmax + 128 * kProducer <= kThreads * kLaunch,
                  "register split exceeds the launch allocation");
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive on `bar` from the threads where `pred` holds, without a branch.
__device__ __forceinline__ void mbar_arrive_if(uint64_t* bar, bool pred) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}"
                 ::"r"(smem_u32(bar)), "r"((uint32_t)pred) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the phase with the given parity has completed.  Returns false
// if the CTA's abort flag is up or the wait ran past kWaitLimitNs (then it
// raises the flag and records the timeout).  After a few unsuccessful polls
// the waiting thread sleeps between polls, so that a warp waiting for a long
// time (the producer and MMA-issuing warps) does not take issue slots from
// the softmax warps of its SM sub-partition.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (it > 2) __nanosleep(it > 64 ? 64 : 16);
        if ((it & 31u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit_ns || it > (1u << 30)) {
                *abort_flag = 1;
                record_status(kStatusTimeout);
                return false;
            }
        }
    }
}

// Tile load from a 4-D map (x = element within a row, y = row, z = head,
// w = batch), completing on `bar`.  x is always 0 here (whole rows).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                            int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w),
          "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit inputs (the type is in idesc), fp32 accumulation.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A (M x K 16-bit, K-major) read from TMEM.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// 32 consecutive TMEM columns of this thread's lane -> 32 registers.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 16 or 8 consecutive TMEM columns of this thread's lane -> registers (the O
// share of a row when it is narrower than 32 columns).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 8 || N == 16 || N == 32, "8, 16 or 32 columns");
    if constexpr (N == 32) {
        tmem_ld32(taddr, r);
    } else if constexpr (N == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
    } else {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
    }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[N]) {
    static_assert(N == 8 || N == 16 || N == 32, "8, 16 or 32 columns");
    if constexpr (N == 32) {
        tmem_st32(taddr, r);
    } else if constexpr (N == 16) {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
            "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
            ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
              "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
            : "memory");
    } else {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                     ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                       "r"(r[7])
                     : "memory");
    }
}

// Shared-memory matrix descriptor of tcgen05: start address, leading and
// stride byte offsets (16-byte units), descriptor version 1, layout type.
constexpr uint32_t kLayoutSw128 = 2, kLayoutSw64 = 4, kLayoutSw32 = 6;

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(layout & 7u) << 61;
    return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, A and B
// both of the type `fmt` (0 = fp16, 1 = bf16; never mixed), A K-major, B
// K-major or MN-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool b_mn_major, uint32_t fmt) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// The 16-bit I/O element types.  kFmt: operand format of kind::f16.  kPBias:
// the exponentials are taken against (running max - kPBias), so the weights P
// lie below 2^(kPBias + 8): fp16 (largest finite 65504) gains 7 binades at
// the small end (values below 2^-24 flush to zero there), bf16 needs none.
template <typename E> struct Elem;
template <> struct Elem<__nv_bfloat16> {
    static constexpr uint32_t kFmt = 1;
    static constexpr float kPBias = 0.f;
    static constexpr CUtensorMapDataType kMapType = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};
template <> struct Elem<__half> {
    static constexpr uint32_t kFmt = 0;
    static constexpr float kPBias = 7.f;
    static constexpr CUtensorMapDataType kMapType = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
};

// 2^x for a pair of arguments on the FMA pipe instead of the MUFU unit.
// Range reduction: n = round(x) by adding 1.5 * 2^23 (the addition rounds x
// to an integer held in the low mantissa bits of t), f = x - n in [-1/2, 1/2]
// exactly; 2^f from the cubic c0 + f (c1 + f (c2 + f c3)), the minimax
// approximation of 2^f on [-1/2, 1/2] for relative error, fitted by the Remez
// exchange algorithm (max relative error 7.5e-5; exp2_poly.py); then 2^n is
// applied by adding n to the exponent field (t's bits shifted left by 23 are
// n << 23).  Arguments below -120 are clamped there: such weights (< 2^-120)
// cannot matter next to the row's largest weight, which is >= 1.
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

__device__ __forceinline__ float2 ex2_fma_pair(float2 x) {
    x.x = fmaxf(x.x, -120.f);
    x.y = fmaxf(x.y, -120.f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
    const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 q = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
    q = __ffma2_rn(q, f, make_float2(kExp2C1, kExp2C1));
    q = __ffma2_rn(q, f, make_float2(kExp2C0, kExp2C0));
    return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// Share of the exponentials that run on the FMA pipe instead of the MUFU unit:
// this many column pairs out of every 64, spread evenly along the row (pair i
// when (i * share) mod 64 falls in the top `share` residues), so that each
// stretch of the row keeps both pipes busy.
constexpr int kFmaExpPairsPer64 = 16;
__host__ __device__ constexpr bool fma_exp_pair(int i) {
    return (i * kFmaExpPairsPer64) % 64 >= 64 - kFmaExpPairsPer64;
}

// max(a, b, c) in one instruction (three-input max.f32)
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}



// ------------------------------------------------------------------ kernel parameters

// Element strides of a tensor of D-element rows: between consecutive rows,
// heads and batch elements.
struct RowStrides {
    int64_t row, h, b;
};
inline RowStrides contiguous_rows(int rows, int H, int D) {
    return {D, (int64_t)rows * D, (int64_t)H * rows * D};
}

enum Mode { kSplit = 0, kDecode = 1 };

struct Params {
    int mode;             // Mode
    int B, H;
    int M, N;             // latents, tokens
    int kv_rows;          // rows of the key/value tensors per (b, h) (N in split mode, M in decode)
    int kv_tiles;         // ceil(kv_rows / KT)
    int q_shared;         // the query tensor is [H, rows, D], shared over the batch (map batch coordinate 0)
    int k_shared;         // the key tensor is [H, rows, D]
    int kv_same;          // values are the keys (synthesis): load one tile per stage
    int interleave;       // warpgroups share one query tile and take the key/value tiles round-robin
    int row_groups;       // split mode: query-row groups per (b, h) (128 rows, or 128 NW when not interleaved)
    int chunks;           // split mode: token chunks per (b, h)
    int chunk_tiles;      // split mode: KT-token tiles per chunk
    int q_groups;         // decode mode: (128 NW)-token query groups per (b, h)
    int items;
    float scale_log2;
    float* part_O;        // split: [parts][B*H][M][D]
    float2* part_ml;      // split: [parts][B*H][M]
    int tok_heads_inner;  // the token tensor's map is ordered (D, H, rows, B): [B,N,H,D] layout
    void* y;              // decode: token rows in E, addressed by the strides below (NULL: not written)
    int64_t y_row, y_h, y_b;   // decode: element strides of y between tokens, heads, batch elements
    float2* tok_stats;    // decode, optional: per token (log-sum-exp in log2 units, <dy, y>) at
                          // tok_stats[(b*H + h)*tok_stats_stride + n] (kept for the backward)
    int64_t tok_stats_stride;
    const void* dy;       // decode with tok_stats: the gradient of y, in E with y's strides
};

struct Item {
    int bh, h;
    int qb, kb, vb;       // batch coordinate of the query, key and value maps (0 for a shared tensor)
    int qrow0;            // first query row of the item
    int t_begin, t_end;   // key/value tile range
    int part;             // split mode: partial index of warpgroup 0 (interleaved: NW c, else c)
};

template <int NW, int MODE>
__device__ __forceinline__ Item decode_item(const Params& p, int item) {
    Item it;
    if constexpr (MODE == kSplit) {
        const int g = item % p.row_groups;
        const int rest = item / p.row_groups;
        const int c = rest % p.chunks;
        it.bh = rest / p.chunks;
        it.qrow0 = g * (p.interleave ? kQTile : NW * kQTile);
        it.t_begin = c * p.chunk_tiles;
        it.t_end = min(p.kv_tiles, it.t_begin + p.chunk_tiles);
        it.part = p.interleave ? NW * c : c;
    } else {
        const int gi = item % p.q_groups;
        it.bh = item / p.q_groups;
        it.qrow0 = gi * NW * kQTile;
        it.t_begin = 0;
        it.t_end = p.kv_tiles;
        it.part = 0;
    }
    it.h = it.bh % p.H;
    const int b = it.bh / p.H;
    it.qb = p.q_shared ? 0 : b;
    it.kb = p.k_shared ? 0 : b;
    it.vb = b;
    return it;
}

// Shared-memory plan: QS query slots of NW [128 x D] tiles, NST stages of a
// [KT x D] key tile and value tile, then the barriers and, with the score
// columns split between CS warps per row (CS = 2), the exchange area of their
// half-row values: [NW row tiles][4 lane quarters][2 phases][CS][32 lanes] fp32.
template <int D, int NW, int KT, int NST, int QS, int CS = 1>
struct Smem {
    static constexpr int kQTileBytes = kQTile * D * 2;
    static constexpr int kKVTileBytes = KT * D * 2;
    static constexpr int kQ = 0;
    static constexpr int kKV = kQ + QS * NW * kQTileBytes;
    static constexpr int kBar = kKV + NST * 2 * kKVTileBytes;
    // kv_full[NST], kv_empty[NST], q_full[QS], q_empty[QS], sfull, sfree, pfull, pfree, drain [NW each],
    // with CS = 2 one exchange barrier per (row tile, lane quarter) [4 NW]
    static constexpr int kNumBars = 2 * NST + 2 * QS + 5 * NW + (CS > 1 ? 4 * NW : 0);
    static constexpr int kX = (kBar + kNumBars * 8 + 15) / 16 * 16;
    static constexpr int kXBytes = CS > 1 ? NW * 4 * 2 * CS * 32 * 4 : 0;
    static constexpr int kMisc = kX + kXBytes;                      // tmem base (u32), abort flag (int)
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kLaunchBytes = kBytes + 1024;              // + alignment slack
};

template <int D, int NW, int KT>
struct Layout {
    // A [rows x D] 16-bit tile is stored as D/64 column blocks of [rows x 64]
    // when D = 128 (a swizzle atom spans at most 128 bytes), else as one block;
    // every block has rows of kRowBytes, swizzled by the same amount.
    static constexpr int kBlocks = D > 64 ? D / 64 : 1;
    static constexpr uint32_t kRowBytes = D > 64 ? 128 : D * 2;
    static constexpr uint32_t kType = kRowBytes == 128 ? kLayoutSw128 : (kRowBytes == 64 ? kLayoutSw64 : kLayoutSw32);
    static constexpr uint32_t kSbo = 8 * kRowBytes;                  // 8-row group stride
    static constexpr uint32_t kQBlockBytes = kQTile * kRowBytes;     // one column block of a query tile
    static constexpr uint32_t kKVBlockBytes = KT * kRowBytes;        // one column block of a key/value tile
    // byte offset of the K-step kk (16 columns) of a K-major tile with `block` bytes per column block
    static __device__ __forceinline__ uint32_t kstep(int kk, uint32_t block) {
        return (kk & 3) * 32 + (kk >> 2) * block;
    }
    // TMEM: O accumulators at least 32 columns apart so that 32-column TMEM
    // loads/stores of one never touch another's
    static constexpr int kOStride = D < 32 ? 32 : D;
    static constexpr int kOCol = NW * KT;
    static constexpr int kPCol = kOCol + NW * kOStride;
    static_assert(kPCol + NW * (KT / 2) <= 512, "TMEM plan exceeds 512 columns");
    static constexpr int kChunks = KT / 32;                          // 32-column score chunks per row
    static constexpr int kPairs = KT / 2;                            // column pairs per row
};

// ------------------------------------------------------------------ the kernel

template <typename E, int D, int NW, int KT, int NST, int QS, int MODE, int CS>
__global__ void __launch_bounds__(Regs<NW * CS>::kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
            const __grid_constant__ CUtensorMap map_v, const Params p) {
    static_assert(D == 16 || D == 32 || D == 64 || D == 128, "tcgen05 path covers D in {16, 32, 64, 128}");
    static_assert(KT == 64 || KT == 128, "key/value tiles of 64 or 128 rows");
    static_assert(NW >= 1 && NW <= 3, "the producer warpgroup holds one TMA warp and NW MMA warps");
    static_assert(NST >= 3, "at least three key/value stages");
    static_assert(CS == 1 || CS == 2, "one or two warps per score row");
    // Interleaved mode (launch_attn refuses it unless NW divides NST): warpgroup w owns stages [w R, w R + R) and consumes them in
    // order, so no consumer can wait on a stage two fills ahead (a parity wait
    // cannot tell phase k+1 from phase k-1).  Shared mode: one ring of NST stages
    // that every warpgroup consumes in order.
    constexpr int R = NST / NW;
    using SM = Smem<D, NW, KT, NST, QS, CS>;
    using LY = Layout<D, NW, KT>;
    constexpr int kSoftmaxWarps = 4 * NW * CS;
    constexpr int kTmaWarp = kSoftmaxWarps;
    constexpr int kMmaWarp0 = kSoftmaxWarps + 1;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
    uint64_t* kv_full = bars;
    uint64_t* kv_empty = bars + NST;
    uint64_t* q_full = bars + 2 * NST;
    uint64_t* q_empty = q_full + QS;
    uint64_t* sfull = q_empty + QS;
    uint64_t* sfree = sfull + NW;
    uint64_t* pfull = sfree + NW;
    uint64_t* pfree = pfull + NW;
    uint64_t* drain = pfree + NW;
    uint64_t* xbar = drain + NW;                 // CS = 2: [NW][4]
    float* xval = reinterpret_cast<float*>(smem + SM::kX);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        // a key/value stage is released by every warpgroup that consumes it;
        // a query slot by every warpgroup
        for (int i = 0; i < NST; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], p.interleave ? 1 : NW); }
        for (int i = 0; i < QS; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], NW); }
        // the softmax side of row tile w arrives once per warp (lane 0): 4 CS warps
        for (int w = 0; w < NW; ++w) {
            mbar_init(&sfull[w], 1);
            mbar_init(&sfree[w], 4 * CS);
            mbar_init(&pfull[w], 4 * CS);
            mbar_init(&pfree[w], 1);
            mbar_init(&drain[w], 1);
        }
        // a column-split exchange completes when every lane of both warps has arrived
        if (CS > 1)
            for (int i = 0; i < 4 * NW; ++i) mbar_init(&xbar[i], 32 * CS);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tensormap(&map_q);
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
    }
    if (warp == kMmaWarp0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int q_tiles = p.interleave ? 1 : NW;                         // query tiles per item
    // the set-up above overlaps the previous kernel's tail; global memory is
    // touched only after it has completed
    pdl_wait();
    pdl_launch_dependents();

    if (warp >= kSoftmaxWarps) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Regs<NW * CS>::kProducer));
      if (warp == kTmaWarp) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t kv_load = 0, q_load = 0, wg_load[NW] = {};
            int kv_last_phase[NST], q_last_phase[QS];
            for (int i = 0; i < NST; ++i) kv_last_phase[i] = -1;
            for (int i = 0; i < QS; ++i) q_last_phase[i] = -1;
            const uint32_t kv_bytes = (p.kv_same ? 1 : 2) * SM::kKVTileBytes;
            const uint32_t q_bytes = q_tiles * SM::kQTileBytes;
            bool ok = true;
            for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
                const Item it = decode_item<NW, MODE>(p, item);
                const int slot = q_load % QS;
                ok = mbar_wait(&q_empty[slot], ((q_load / QS) & 1) ^ 1, abort_flag);
                if (!ok) break;
                mbar_expect_tx(&q_full[slot], q_bytes);
                uint8_t* qdst = smem + SM::kQ + slot * NW * SM::kQTileBytes;
                for (int qt = 0; qt < q_tiles; ++qt) {
                    const int qrow = it.qrow0 + qt * kQTile;
#pragma unroll
                    for (int cb = 0; cb < LY::kBlocks; ++cb) {
                        uint8_t* dst = qdst + qt * SM::kQTileBytes + cb * LY::kQBlockBytes;
                        if (MODE == kDecode && p.tok_heads_inner)  // token queries, [B,N,H,D]
                            tma_load_4d(dst, &map_q, &q_full[slot], cb * 64, it.h, qrow, it.qb);
                        else
                            tma_load_4d(dst, &map_q, &q_full[slot], cb * 64, qrow, it.h, it.qb);
                    }
                }
                q_last_phase[slot] = (q_load / QS) & 1;
                ++q_load;
                for (int t = it.t_begin; t < it.t_end; ++t) {
                    int st;
                    uint32_t fill;                     // fills of this stage before this one
                    if (p.interleave) {
                        const int ow = (t - it.t_begin) % NW;
                        st = ow * R + (int)(wg_load[ow] % R);
                        fill = wg_load[ow] / R;
                        ++wg_load[ow];
                    } else {
                        st = kv_load % NST;
                        fill = kv_load / NST;
                    }
                    ok = mbar_wait(&kv_empty[st], (fill & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    mbar_expect_tx(&kv_full[st], kv_bytes);
                    uint8_t* kdst = smem + SM::kKV + st * 2 * SM::kKVTileBytes;
                    const bool hi = MODE == kSplit && p.tok_heads_inner;   // token keys/values, [B,N,H,D]
#pragma unroll
                    for (int cb = 0; cb < LY::kBlocks; ++cb) {
                        tma_load_4d(kdst + cb * LY::kKVBlockBytes, &map_k, &kv_full[st], cb * 64,
                                    hi ? it.h : t * KT, hi ? t * KT : it.h, it.kb);
                        if (!p.kv_same)
                            tma_load_4d(kdst + SM::kKVTileBytes + cb * LY::kKVBlockBytes, &map_v, &kv_full[st],
                                        cb * 64, hi ? it.h : t * KT, hi ? t * KT : it.h, it.vb);
                    }
                    kv_last_phase[st] = fill & 1;
                    ++kv_load;
                }
            }
            if (!ok) {
                // Let the copies already issued land before the CTA exits (bounded):
                // the last phase issued on each barrier completes when its bytes arrive.
                const unsigned long long t0 = globaltimer_ns();
                for (int s = 0; s < NST; ++s)
                    while (kv_last_phase[s] >= 0 && !mbar_try_wait(&kv_full[s], kv_last_phase[s]) &&
                           globaltimer_ns() - t0 < 100000000ull) {
                    }
                for (int s = 0; s < QS; ++s)
                    while (q_last_phase[s] >= 0 && !mbar_try_wait(&q_full[s], q_last_phase[s]) &&
                           globaltimer_ns() - t0 < 100000000ull) {
                    }
            }
        }
      } else if (warp >= kMmaWarp0 && warp < kMmaWarp0 + NW) {
        // ---------------------------------------------------------- MMA issuers
        // Warp kMmaWarp0 + w issues for softmax warpgroup w, so the warpgroups'
        // pipelines never wait on each other's softmax.
        if (lane == 0) {
            const int w = warp - kMmaWarp0;
            constexpr uint32_t idesc_s = make_idesc(kQTile, KT, false, Elem<E>::kFmt);   // S = Q K^T: [128 q x KT kv]
            constexpr uint32_t idesc_o = make_idesc(kQTile, D, true, Elem<E>::kFmt);     // O += P V: [128 q x D], V MN-major
            const int tstep = p.interleave ? NW : 1;
            const int tfirst = p.interleave ? w : 0;
            // This warpgroup's jobs: the key/value tiles it consumes, item by item.
            // One cursor over the stream issues the score MMAs one job ahead of the
            // value MMAs; what a value MMA needs of its job (the key/value stage,
            // whether it starts the item's accumulator) is kept from its score
            // MMA in a two-entry record, so the issuer needs few registers.
            struct Cursor {
                int item, t, njobs;
                bool valid;
                Item info;
                uint32_t tiles_before, item_count;
            };
            bool ok = true;
            // Settles on the next item (from c.item on) that has a job for this
            // warpgroup.  An item without one still takes part in freeing its
            // query slot, after the slot's load has landed (so the release is
            // counted in the right phase).
            auto settle = [&](Cursor& c) {
                while (c.item < p.items) {
                    c.info = decode_item<NW, MODE>(p, c.item);
                    c.t = c.info.t_begin + tfirst;
                    c.njobs = 0;
                    if (c.t < c.info.t_end) {
                        c.valid = true;
                        return;
                    }
                    if (ok) {
                        const int slot = c.item_count % QS;
                        ok = mbar_wait(&q_full[slot], (c.item_count / QS) & 1, abort_flag);
                        if (ok) umma_commit(&q_empty[slot]);
                    }
                    c.tiles_before += c.info.t_end - c.info.t_begin;
                    ++c.item_count;
                    c.item += gridDim.x;
                }
                c.valid = false;
            };
            auto first = [&](Cursor& c) {
                c.item = blockIdx.x;
                c.tiles_before = 0;
                c.item_count = 0;
                settle(c);
            };
            auto next = [&](Cursor& c) {
                ++c.njobs;
                c.t += tstep;
                if (c.t < c.info.t_end) return;
                c.tiles_before += c.info.t_end - c.info.t_begin;
                ++c.item_count;
                c.item += gridDim.x;
                settle(c);
            };
            // stage and fill count of the cursor's tile: this warpgroup's own ring in
            // interleaved mode (its j-th tile), else the shared ring (global tile count)
            auto stage_of = [&](const Cursor& c, uint32_t j, uint32_t& fill) -> int {
                if (p.interleave) {
                    fill = j / R;
                    return w * R + (int)(j % R);
                }
                const uint32_t g = c.tiles_before + (c.t - c.info.t_begin);
                fill = g / NST;
                return (int)(g % NST);
            };
            uint32_t s_issued = 0, pv_issued = 0;
            // the two outstanding jobs' stages and "first job of its item" flags (entry = job parity)
            int job_st0 = 0, job_st1 = 0;
            bool job_first0 = false, job_first1 = false;
            auto issue_s = [&](const Cursor& c) -> bool {
                const int slot = c.item_count % QS;
                if (c.njobs == 0 && !mbar_wait(&q_full[slot], (c.item_count / QS) & 1, abort_flag)) return false;
                uint32_t fill;
                const int st = stage_of(c, s_issued, fill);
                if (!mbar_wait(&kv_full[st], fill & 1, abort_flag)) return false;
                if (!mbar_wait(&sfree[w], (s_issued & 1) ^ 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t qaddr = smem_u32(smem + SM::kQ + slot * NW * SM::kQTileBytes +
                                                (p.interleave ? 0 : w * SM::kQTileBytes));
                const uint32_t kaddr = smem_u32(smem + SM::kKV + st * 2 * SM::kKVTileBytes);
                const uint32_t d_tmem = tmem + w * KT;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = smem_desc(qaddr + LY::kstep(kk, LY::kQBlockBytes), 16, LY::kSbo, LY::kType);
                    const uint64_t bd = smem_desc(kaddr + LY::kstep(kk, LY::kKVBlockBytes), 16, LY::kSbo, LY::kType);
                    umma_f16(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sfull[w]);
                if (s_issued & 1) {
                    job_st1 = st;
                    job_first1 = c.njobs == 0;
                } else {
                    job_st0 = st;
                    job_first0 = c.njobs == 0;
                }
                ++s_issued;
                // this warpgroup's last score MMA of the item releases its share of the query slot
                if (c.t + tstep >= c.info.t_end) umma_commit(&q_empty[slot]);
                return true;
            };
            auto issue_pv = [&]() -> bool {
                if (!mbar_wait(&pfull[w], pv_issued & 1, abort_flag)) return false;
                tc_fence_after();
                const int st = (pv_issued & 1) ? job_st1 : job_st0;
                const bool first_job = (pv_issued & 1) ? job_first1 : job_first0;
                const uint8_t* vbase = smem + SM::kKV + st * 2 * SM::kKVTileBytes + (p.kv_same ? 0 : SM::kKVTileBytes);
                const uint32_t vaddr = smem_u32(vbase);
                const uint32_t d_tmem = tmem + LY::kOCol + w * LY::kOStride;
                const uint32_t p_tmem = tmem + LY::kPCol + w * (KT / 2);
#pragma unroll
                for (int kk = 0; kk < KT / 16; ++kk) {
                    // A = P in TMEM: 16 key/value columns = 8 columns of packed pairs per step
                    // B = V tile [KT kv x D], D contiguous: MN-major; 16 kv rows per step
                    // (D fits one swizzle atom along MN, so the leading offset is never used)
                    // (D = 128: the two 64-column blocks are the MN atoms, kKVBlockBytes apart)
                    const uint64_t bd = smem_desc(vaddr + kk * 16 * LY::kRowBytes, LY::kKVBlockBytes,
                                                  LY::kSbo, LY::kType);
                    umma_f16_tmem_a(d_tmem, p_tmem + kk * 8, bd, idesc_o, (first_job && kk == 0) ? 0u : 1u);
                }
                umma_commit(&pfree[w]);
                ++pv_issued;
                umma_commit(&kv_empty[st]);     // this warpgroup is done with the stage
                return true;
            };
            Cursor sc;
            first(sc);
            if (sc.valid && ok) {
                ok = issue_s(sc);
                next(sc);
            }
            while (pv_issued < s_issued && ok) {
                if (sc.valid) {
                    ok = issue_s(sc);
                    if (!ok) break;
                    next(sc);
                }
                ok = issue_pv();
            }
            // drain: wait until every issued MMA has completed before TMEM is
            // released; if that runs out, report it (the outputs are then undefined)
            umma_commit(&drain[w]);
            const unsigned long long t0 = globaltimer_ns();
            bool drained = false;
            while (!(drained = mbar_try_wait(&drain[w], 0)) && globaltimer_ns() - t0 < kWaitLimitNs) {
            }
            if (!drained) {
                *abort_flag = 1;
                record_status(kStatusTimeout);
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Regs<NW * CS>::kSoftmax));
        // ---------------------------------------------------------- softmax warpgroups
        // Softmax warpgroup g = warp / 4 serves row tile wg = g / CS and takes the
        // column share `half` = g % CS of each job: CW = KT / CS score columns, the
        // matching CW / 2 columns of P and D / CS columns of O.  With CS = 2 the
        // two warps on one TMEM
        // lane quarter exchange their half-row maxima through shared memory every
        // job, so both take the weights against the same running maximum, and
        // their half-row sums at the end of an item.
        constexpr int CW = KT / CS;
        constexpr int kCChunks = CW / 32;
        constexpr int kPSt = CW / 2 < 32 ? CW / 2 : 32;         // packed P columns per TMEM store
        constexpr int kPChunks = CW / 2 / kPSt;
        constexpr int kOCols = D / CS;                          // this share's O columns
        constexpr int kOLd = kOCols < 32 ? kOCols : 32;         // O columns per TMEM load
        constexpr int kOChunks = kOCols / kOLd;
        const int g = warp >> 2;
        const int wg = g / CS;
        const int half = g % CS;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + wg * KT + half * CW;
        const uint32_t tO = tmem + lane_base + LY::kOCol + wg * LY::kOStride + half * kOCols;
        const uint32_t tP = tmem + lane_base + LY::kPCol + wg * (KT / 2) + half * (CW / 2);
        const float sl2 = p.scale_log2;
        const int tstep = p.interleave ? NW : 1;
        const int tfirst = p.interleave ? wg : 0;
        uint32_t sfull_waits = 0, pfree_waits = 0, jobs_done = 0, xph = 0;
        bool ok = true;
        // CS = 2: the other share's value of this thread's row (both shares call
        // this in the same order: once per job and once per finished item)
        uint64_t* my_xbar = xbar + (wg * 4 + wq);
        float* my_xval = xval + (wg * 4 + wq) * 2 * CS * 32;
        auto exchange = [&](float v) -> float {
            if constexpr (CS == 1) {
                return v;
            } else {
                float* slot = my_xval + (xph & 1) * CS * 32;
                slot[half * 32 + lane] = v;
                mbar_arrive(my_xbar);
                if (!mbar_wait(my_xbar, xph & 1, abort_flag)) ok = false;
                ++xph;
                return slot[(half ^ 1) * 32 + lane];
            }
        };
        // Item outputs from this thread's share of its O row (o == nullptr: the
        // warpgroup had no job in the item); value e of the share is o[e / kOLd][e % kOLd].
        auto ov = [](const uint32_t (*o)[kOLd], int e) { return __uint_as_float(o[e / kOLd][e % kOLd]); };
        auto write_outputs = [&](const Item& it, int njobs, float m, float l, const uint32_t (*o)[kOLd]) {
            if constexpr (MODE == kSplit) {
                const int r = it.qrow0 + (p.interleave ? 0 : wg * kQTile) + row;
                const int part = p.interleave ? it.part + wg : it.part;
                if (r < p.M) {
                    const int64_t ridx = ((int64_t)part * p.B * p.H + it.bh) * p.M + r;
                    if (half == 0) p.part_ml[ridx] = make_float2(njobs > 0 ? m : -INFINITY, l);
                    float* dst = p.part_O + ridx * D + half * kOCols;
                    if constexpr (kOCols >= 4) {
#pragma unroll
                        for (int i = 0; i < kOCols / 4; ++i)
                            reinterpret_cast<float4*>(dst)[i] =
                                o ? make_float4(ov(o, 4 * i), ov(o, 4 * i + 1), ov(o, 4 * i + 2), ov(o, 4 * i + 3))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
            } else {
                // decode: this share's columns of y (every lane of both shares takes
                // part in the <dy, y> exchange, also for rows past N)
                const int n = it.qrow0 + wg * kQTile + row;
                const bool valid_row = n < p.N && o != nullptr;
                const float inv = 1.f / l;
                const int64_t off = (int64_t)(it.bh / p.H) * p.y_b + (int64_t)it.h * p.y_h + (int64_t)n * p.y_row +
                                    half * kOCols;
                static_assert(kOCols % 8 == 0, "16-byte stores of y");
                if (valid_row && p.y) {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<E*>(p.y) + off);
#pragma unroll
                    for (int i = 0; i < kOCols / 8; ++i) {
                        const int e = 8 * i;
                        dst[i] = make_uint4(pack2<E>(ov(o, e + 0) * inv, ov(o, e + 1) * inv),
                                            pack2<E>(ov(o, e + 2) * inv, ov(o, e + 3) * inv),
                                            pack2<E>(ov(o, e + 4) * inv, ov(o, e + 5) * inv),
                                            pack2<E>(ov(o, e + 6) * inv, ov(o, e + 7) * inv));
                    }
                }
                if (__builtin_expect(p.tok_stats != nullptr, 0)) {
                    // the backward's per-token statistics: the softmax's log-sum-exp
                    // (log2 units, against the same running max as l) and <dy, y>
                    // (0 when no dy is given: a forward that saves its state)
                    float dsum = 0.f;
                    if (valid_row && p.dy) {
                        const uint4* g4 = reinterpret_cast<const uint4*>(static_cast<const E*>(p.dy) + off);
#pragma unroll
                        for (int i = 0; i < kOCols / 8; ++i) {
                            const uint4 v = g4[i];
                            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 g2 = unpack2<E>(w4[e]);
                                dsum = fmaf(g2.x, ov(o, 8 * i + 2 * e), dsum);
                                dsum = fmaf(g2.y, ov(o, 8 * i + 2 * e + 1), dsum);
                            }
                        }
                    }
                    if constexpr (CS > 1) dsum += exchange(dsum);
                    if (valid_row && half == 0)
                        p.tok_stats[(int64_t)it.bh * p.tok_stats_stride + n] = make_float2(m + log2f(l), dsum * inv);
                }
            }
        };
        // this share of the O row of the finished item -> outputs (every value MMA
        // of the item has completed)
        auto flush = [&](const Item& it, int njobs, float m, float l) {
            uint32_t o[kOChunks][kOLd];
#pragma unroll
            for (int c = 0; c < kOChunks; ++c) tmem_ld_cols<kOLd>(tO + c * kOLd, o[c]);
            tmem_wait_ld();
            write_outputs(it, njobs, m, l, o);
        };
        // Decode: the epilogue of an item (a few jobs long) is deferred into the
        // next item's first job, so its last value MMA finishes while the next
        // exponentials are computed and its O row is read just before the next
        // value MMA overwrites it.  Split passes (items of hundreds of jobs):
        // the epilogue runs at the end of the item, which keeps the job loop
        // free of the pending item's state.
        constexpr bool kDefer = MODE == kDecode;
        bool pend = false;
        Item pend_it{};
        int pend_jobs = 0;
        float pend_m = 0.f, pend_l = 0.f;
        for (int item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
            const Item it = decode_item<NW, MODE>(p, item);
            float m_run = -INFINITY, l_run = 0.f;
            int njobs = 0;
            for (int t = it.t_begin + tfirst; t < it.t_end; t += tstep) {
                if (!mbar_wait(&sfull[wg], sfull_waits & 1, abort_flag)) { ok = false; break; }
                ++sfull_waits;
                tc_fence_after();
                uint32_t sr[kCChunks][32];
#pragma unroll
                for (int c = 0; c < kCChunks; ++c) tmem_ld32(tS + c * 32, sr[c]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                mbar_arrive_if(&sfree[wg], lane == 0);

                // key/value rows of this tile that exist, counted from this share's first column
                const int valid = p.kv_rows - t * KT - half * CW;
                if (__builtin_expect(valid < CW, 0)) {            // ragged last tile only (warp-uniform)
#pragma unroll
                    for (int c = 0; c < kCChunks; ++c)
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c * 32 + j >= valid) sr[c][j] = __float_as_uint(-INFINITY);
                }
                // row max: one chain of 3-input maxima per 32-column chunk (a tree of
                // maxima measured slower here), then the other share's (CS = 2)
                float mc[kCChunks];
#pragma unroll
                for (int c = 0; c < kCChunks; ++c) {
                    mc[c] = __uint_as_float(sr[c][0]);
#pragma unroll
                    for (int j = 1; j < 31; j += 2)
                        mc[c] = max3f(mc[c], __uint_as_float(sr[c][j]), __uint_as_float(sr[c][j + 1]));
                    mc[c] = fmaxf(mc[c], __uint_as_float(sr[c][31]));
                }
                float mx = mc[0];
#pragma unroll
                for (int c = 1; c < kCChunks; ++c) mx = fmaxf(mx, mc[c]);
                if constexpr (CS > 1) {
                    mx = fmaxf(mx, exchange(mx));
                    if (!ok) break;
                }
                const float m_new = fmaxf(m_run, mx * sl2 - Elem<E>::kPBias);
                float factor = 1.f;
                const bool resc = m_new > m_run + kRescaleLog2;
                if (__builtin_expect(resc, 0)) {
                    factor = ex2_mufu(m_run - m_new);
                    m_run = m_new;
                }
                // exponent arguments in pairs (packed fp32 FMA), row sum in packed chains
                const float2 sl2v = make_float2(sl2, sl2);
                const float2 negm = make_float2(-m_run, -m_run);
                float2 acc[kCChunks];
                // packed weight column q (this share's columns 2 q, 2 q + 1) -> pk[q / kPSt][q % kPSt]
                uint32_t pk[kPChunks][kPSt];
#pragma unroll
                for (int c = 0; c < kCChunks; ++c) {
                    acc[c] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float2 sv = make_float2(__uint_as_float(sr[c][2 * j]), __uint_as_float(sr[c][2 * j + 1]));
                        const float2 xv = __ffma2_rn(sv, sl2v, negm);
                        const float2 pv = fma_exp_pair(half * (CW / 2) + c * 16 + j)
                                              ? ex2_fma_pair(xv)
                                              : make_float2(ex2_mufu(xv.x), ex2_mufu(xv.y));
                        acc[c] = __fadd2_rn(acc[c], pv);
                        pk[(c * 16 + j) / kPSt][(c * 16 + j) % kPSt] = pack2<E>(pv.x, pv.y);
                    }
                }
                float2 asum = acc[0];
#pragma unroll
                for (int c = 1; c < kCChunks; ++c) asum = __fadd2_rn(asum, acc[c]);
                l_run = l_run * factor + (asum.x + asum.y);

                // the previous value MMA of this row tile must be done before P and O are touched
                while (pfree_waits < jobs_done) {
                    if (!mbar_wait(&pfree[wg], pfree_waits & 1, abort_flag)) { ok = false; break; }
                    ++pfree_waits;
                }
                if (!ok) break;
                tc_fence_after();
                // this share of the P row -> TMEM (this thread's lane, CW/2 columns of packed pairs)
#pragma unroll
                for (int h = 0; h < kPChunks; ++h) tmem_st_cols<kPSt>(tP + h * kPSt, pk[h]);
                // Rare work on O, after P is out of the registers and before the
                // value MMA of this job adds to O: the previous item's O row (first
                // job of a decode item), or the O rescale of a grown running max
                // (each share rescales its own O columns).
                if constexpr (kDefer) {
                    if (__builtin_expect(pend, 0)) {
                        flush(pend_it, pend_jobs, pend_m, pend_l);
                        pend = false;
                    }
                }
                if (__builtin_expect(__any_sync(0xffffffffu, resc && njobs > 0), 0)) {
                    const float f = njobs > 0 ? factor : 1.f;
#pragma unroll
                    for (int c = 0; c < kOChunks; ++c) {
                        uint32_t o[kOLd];
                        tmem_ld_cols<kOLd>(tO + c * kOLd, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < kOLd; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                        tmem_st_cols<kOLd>(tO + c * kOLd, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                mbar_arrive_if(&pfull[wg], lane == 0);
                ++jobs_done;
                ++njobs;
            }
            if (!ok) break;

            // ---------------- end of the item: its epilogue (deferred in the decode)
            if (njobs == 0) {
                write_outputs(it, 0, m_run, l_run, nullptr);
            } else if constexpr (kDefer) {
                pend = true;
                pend_it = it;
                pend_jobs = njobs;
                pend_m = m_run;
                pend_l = CS > 1 ? l_run + exchange(l_run) : l_run;
                if (!ok) break;
            } else {
                const float l_row = CS > 1 ? l_run + exchange(l_run) : l_run;
                if (!ok) break;
                while (pfree_waits < jobs_done) {
                    if (!mbar_wait(&pfree[wg], pfree_waits & 1, abort_flag)) { ok = false; break; }
                    ++pfree_waits;
                }
                if (!ok) break;
                tc_fence_after();
                flush(it, njobs, m_run, l_row);
            }
        }
        if (kDefer && ok && pend) {
            while (pfree_waits < jobs_done) {
                if (!mbar_wait(&pfree[wg], pfree_waits & 1, abort_flag)) { ok = false; break; }
                ++pfree_waits;
            }
            if (ok) {
                tc_fence_after();
                flush(pend_it, pend_jobs, pend_m, pend_l);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// Self-test of the failure path: one thread waits, with a short limit, on an
// mbarrier that nothing arrives at.  The bounded wait gives up, records
// FLAREPP_ERR_TIMEOUT in the device status word and the kernel returns.
__global__ void wait_timeout_selftest(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

// ------------------------------------------------------------------ host side

struct Buffers {
    float* part_O;
    float2* part_ml;
    float* q32;
    void* q16;            // q in E: the MMA operand
    float* z32;
    void* z16;            // z in E
};

struct Problem {
    int B, H, N, M, D;
    RowStrides tok;       // element strides of the token tensors k0, k, v, y
    int chunks, chunk_len;
    float scale_log2;
};

// Kernel configurations: NW softmax warpgroups, KT-row key/value tiles, NST
// key/value stages, QS query slots.  The split passes (synthesis, encode) use
// two warpgroups on 128-row key/value tiles that both consume (each tile read
// from L2 once per 256 latents); the decode uses three warpgroups on 64-row
// latent tiles (more softmax warps per SM sub-partition to hide latency).
template <int D, int NW_, int KT_, bool DECODE = false>
struct Config {
    static constexpr int NW = NW_;
    static constexpr int KT = KT_;
    // D = 128 fits four key/value stages and one query slot (split passes:
    // long items) or three stages and two slots (decode: an item is a few
    // latent tiles, so the next item's query tiles load during the current one)
    static constexpr int NST = NW == 3 ? (D == 64 ? 6 : 9) : (D == 128 ? (DECODE ? 3 : 4) : (D == 64 ? 4 : 6));
    static constexpr int QS = D == 128 && !DECODE ? 1 : 2;
    // split passes on 128-column jobs at D = 64: two softmax warps per row,
    // each taking 64 of the columns (four softmax warps per SM sub-partition;
    // measured 3-4% faster than one warp per row at the 1M-token workload).
    // At D <= 32 the column split (O divided between the shares, no spills)
    // still ran 3-7% slower (40000-token cloud: split launch 0.0416 against
    // 0.0402 ms; 16641-token grid: 0.0249 against 0.0232), and the decode keeps three
    // warpgroups on 64-row latent tiles (on two warpgroups with 128-row tiles
    // and two warps per row it ran 2.0 ms against 1.52).
    static constexpr int CS = !DECODE && KT == 128 && D == 64 ? 2 : 1;
    using SM = Smem<D, NW, KT, NST, QS, CS>;
    // at least 116 KB so that a second CTA (which would block on TMEM) never shares the SM
    static constexpr int kSmemLaunch = SM::kLaunchBytes > 118784 ? SM::kLaunchBytes : 118784;
};
constexpr int kSplitNW = 2, kSplitKT = 128;
constexpr int kDecodeNW = 3, kDecodeKT = 64;

inline bool supported(bool io16, int D, int M) {
    (void)M;
    return io16 && (D == 16 || D == 32 || D == 64 || D == 128);
}

// D = 128 keeps two warpgroups in both passes on 64-row tiles (TMEM: 2 x (64
// score + 128 accumulator + 32 weight columns) = 448 of 512).
inline int split_kt(int D) { return D == 128 ? 64 : kSplitKT; }
inline int decode_nw(int D) { return D == 128 ? 2 : kDecodeNW; }
// latent rows per key/value tile of the decode (the box height of its latent maps)
inline int decode_kt(int D) { return D == 128 ? 64 : kDecodeKT; }

// Split-pass plan.  With one 128-row tile holding all M latents, the two
// warpgroups share it and take the key/value tiles round-robin (interleaved,
// two partial triples per chunk); otherwise each takes its own 128 latents.
inline int kv_tile(int D) { return split_kt(D); }
inline bool interleaved(int M) { return M <= kQTile; }
inline int row_groups(int M) {
    return interleaved(M) ? (M + kQTile - 1) / kQTile : (M + kSplitNW * kQTile - 1) / (kSplitNW * kQTile);
}
inline int parts_per_chunk(int M) { return interleaved(M) ? kSplitNW : 1; }

// Token chunks per (b, h) for the split passes.  With `units` items per
// chunk count step ((b, h) x latent groups) and `tiles` key/value tiles per
// (b, h), c chunks give units*c items in ceil(units*c / sms) waves, each item
// holding ceil(tiles / c) tiles, i.e. that many jobs per warpgroup (divided by
// the warpgroup count when interleaved).  An item costs about two jobs of
// fixed work (query load, first-tile max, epilogue), so the time is about
// waves * (2 + jobs per item); take the cheapest c (the largest on ties).
inline int64_t choose_chunks(int64_t units, int64_t tiles, int sms, int jobs_div) {
    int64_t best_c = 1;
    double best = 1e300;
    for (int64_t c = 1; c <= tiles; ++c) {
        const int64_t per = (tiles + c - 1) / c;
        if (c > 1 && (tiles + per - 1) / per < c) continue;          // same split as a smaller c
        const int64_t waves = (units * c + sms - 1) / sms;
        const double cost = (double)waves * (2.0 + (double)((per + jobs_div - 1) / jobs_div));
        if (cost <= best) {
            best = cost;
            best_c = c;
        }
    }
    return best_c;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 4-D map over a tensor of 16-bit elements, box of box_rows whole rows of one
// (b, h), swizzle = D*2 bytes.  The dimensions are ordered by increasing
// stride: (D, rows, H, B) when a head's rows are contiguous ([B,H,rows,D]),
// (D, H, rows, B) when a row's heads are ([B,rows,H,D]); the kernel passes its
// coordinates in the same order (Params::tok_heads_inner).
inline bool make_map(CUtensorMap* map, CUtensorMapDataType type, const void* base, int rows, int H, int B, int D,
                     const RowStrides& str, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const bool heads_inner = str.h < str.row;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)(heads_inner ? H : rows),
                                (cuuint64_t)(heads_inner ? rows : H), (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)(heads_inner ? str.h : str.row) * 2,
                                   (cuuint64_t)(heads_inner ? str.row : str.h) * 2, (cuuint64_t)str.b * 2};
    // a box holds one column block: all D columns, or 64 of them when D = 128
    const cuuint32_t bx = D > 64 ? 64u : (cuuint32_t)D;
    const cuuint32_t box[4] = {bx, heads_inner ? 1u : (cuuint32_t)box_rows, heads_inner ? (cuuint32_t)box_rows : 1u, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw = bx == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                           : (bx == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    return fn(map, type, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with programmatic stream serialization (the kernel calls pdl_wait()
// before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

inline int sm_count() {
    int dev = 0, n = kNumSMs;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : kNumSMs;
}

template <typename E, int D, int NW, int KT, bool DECODE = false>
int launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const Params& prm,
                cudaStream_t st) {
    using C = Config<D, NW, KT, DECODE>;
    if (prm.interleave && C::NST % C::NW != 0) return 2;      // one stage ring per warpgroup needs NW | NST
    auto kern = attn_kernel<E, D, C::NW, C::KT, C::NST, C::QS, DECODE ? kDecode : kSplit, C::CS>;
    static_assert(C::SM::kLaunchBytes <= 232448, "shared memory plan exceeds 227 KB");
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemLaunch) != cudaSuccess)
        return 3;
    const int grid = prm.items < sm_count() ? prm.items : sm_count();
    return launch_pdl(kern, dim3(grid), dim3(Regs<C::NW * C::CS>::kThreads), C::kSmemLaunch, st, mq, mk, mv, prm) ==
                   cudaSuccess
               ? 0
               : 3;
}

template <typename E, int NW, int KT, bool DECODE>
inline int launch_attn_d(int D, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const Params& prm, cudaStream_t st) {
    switch (D) {
        case 16: return launch_attn<E, 16, NW, KT, DECODE>(mq, mk, mv, prm, st);
        case 32: return launch_attn<E, 32, NW, KT, DECODE>(mq, mk, mv, prm, st);
        case 64: return launch_attn<E, 64, NW, KT, DECODE>(mq, mk, mv, prm, st);
        default: return 2;
    }
}

template <typename E>
inline int launch_split(int D, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const Params& prm, cudaStream_t st) {
    if (D == 128) return launch_attn<E, 128, 2, 64>(mq, mk, mv, prm, st);
    return launch_attn_d<E, kSplitNW, kSplitKT, false>(D, mq, mk, mv, prm, st);
}

template <typename E>
inline int launch_decode(int D, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const Params& prm, cudaStream_t st) {
    if (D == 128) return launch_attn<E, 128, 2, 64, true>(mq, mk, mv, prm, st);
    return launch_attn_d<E, kDecodeNW, kDecodeKT, true>(D, mq, mk, mv, prm, st);
}

template <typename E, int D>
void launch_merge(const MergeParams& mp, int64_t rows, cudaStream_t st) {
    // the attention kernels run with the largest shared-memory carveout; the
    // merge asks for the same so that the SMs are not reconfigured in between
    static const cudaError_t carveout = cudaFuncSetAttribute(
        merge_partials<E, D>, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    (void)carveout;
    launch_pdl(merge_partials<E, D>, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, st, mp);
}

template <typename E>
inline void launch_merge_d(int D, const MergeParams& mp, int64_t rows, cudaStream_t st) {
    switch (D) {
        case 16: launch_merge<E, 16>(mp, rows, st); break;
        case 32: launch_merge<E, 32>(mp, rows, st); break;
        case 64: launch_merge<E, 64>(mp, rows, st); break;
        default: launch_merge<E, 128>(mp, rows, st); break;
    }
}

// The whole FLARE++ forward on the tcgen05 path; `mark(stream)` is called
// before the first launch and after each launch.
template <typename E, typename Mark>
int run(const Problem& pr, const Buffers& bu, const void* q0, const void* q_fixed, const float* gate,
        const void* k0, const void* k, const void* v, void* y, float* q_out, float* z_out, Mark&& mark,
        cudaStream_t st, const FwdExtras& ex = FwdExtras{}) {
    const bool gated = gate != nullptr;
    const int B = pr.B, H = pr.H, N = pr.N, M = pr.M, D = pr.D, BH = B * H;
    // query maps use 128-row boxes, key/value maps the pass's tile height; the
    // token keys k serve as key/value tiles (split) and as query tiles (decode)
    CUtensorMap m_q0, m_qf_q, m_qf_kv, m_q16_q, m_q16_kv, m_z16, m_k0, m_k_kv, m_k_q, m_v;
    const CUtensorMapDataType ty = Elem<E>::kMapType;
    const RowStrides lat1 = contiguous_rows(M, H, D), latb = contiguous_rows(M, H, D), tok = pr.tok;
    bool ok = make_map(&m_qf_q, ty, q_fixed, M, H, 1, D, lat1, kQTile) &&
              make_map(&m_qf_kv, ty, q_fixed, M, H, 1, D, lat1, decode_kt(D)) &&
              make_map(&m_q16_q, ty, bu.q16, M, H, B, D, latb, kQTile) &&
              make_map(&m_q16_kv, ty, bu.q16, M, H, B, D, latb, decode_kt(D)) &&
              make_map(&m_z16, ty, bu.z16, M, H, B, D, latb, decode_kt(D)) &&
              make_map(&m_k_kv, ty, k, N, H, B, D, tok, split_kt(D)) && make_map(&m_k_q, ty, k, N, H, B, D, tok, kQTile) &&
              make_map(&m_v, ty, v, N, H, B, D, tok, split_kt(D));
    if (gated)
        ok = ok && make_map(&m_q0, ty, q0, M, H, 1, D, lat1, kQTile) &&
             make_map(&m_k0, ty, k0, N, H, B, D, tok, split_kt(D));
    if (!ok) return 3;

    const int kv_tiles = (N + split_kt(D) - 1) / split_kt(D);
    const int chunk_tiles = pr.chunk_len / split_kt(D);
    Params sp{};
    sp.mode = kSplit;
    sp.B = B; sp.H = H; sp.M = M; sp.N = N;
    sp.kv_rows = N; sp.kv_tiles = kv_tiles;
    sp.tok_heads_inner = pr.tok.h < pr.tok.row ? 1 : 0;
    sp.interleave = interleaved(M) ? 1 : 0;
    sp.row_groups = row_groups(M);
    sp.chunks = pr.chunks;
    sp.chunk_tiles = chunk_tiles;
    sp.items = BH * pr.chunks * sp.row_groups;
    sp.scale_log2 = pr.scale_log2;
    sp.part_O = bu.part_O;
    sp.part_ml = bu.part_ml;
    const int parts = pr.chunks * parts_per_chunk(M);

    MergeParams mp{};
    mp.part_O = bu.part_O; mp.part_ml = bu.part_ml; mp.chunks = parts;
    mp.B = B; mp.H = H; mp.M = M; mp.q_fixed = q_fixed; mp.gate = gate;
    const int64_t rows = (int64_t)BH * M;

    int rc = 0;
    mark(st);
    if (gated) {
        Params s1 = sp;
        s1.q_shared = 1; s1.k_shared = 0; s1.kv_same = 1;
        rc = launch_split<E>(D, m_q0, m_k0, m_k0, s1, st);
        if (rc) return rc;
        mark(st);
        mp.mode = kMergeSynthesis; mp.out_f32 = bu.q32; mp.out_16 = bu.q16; mp.user_out = q_out;
        mp.q_copy_out = nullptr; mp.lse_out = ex.lse_syn; mp.pregate_out = ex.qdyn;
        launch_merge_d<E>(D, mp, rows, st);
        mark(st);
    }
    Params s2 = sp;
    s2.q_shared = gated ? 0 : 1; s2.k_shared = 0; s2.kv_same = 0;
    rc = launch_split<E>(D, gated ? m_q16_q : m_qf_q, m_k_kv, m_v, s2, st);
    if (rc) return rc;
    mark(st);
    mp.mode = kMergeEncode; mp.out_f32 = bu.z32; mp.out_16 = bu.z16; mp.user_out = z_out;
    mp.q_copy_out = gated ? nullptr : q_out; mp.lse_out = ex.lse_enc; mp.pregate_out = nullptr;
    launch_merge_d<E>(D, mp, rows, st);
    mark(st);
    if (!ex.decode) return cudaGetLastError() == cudaSuccess ? 0 : 3;

    Params dp{};
    dp.mode = kDecode;
    dp.B = B; dp.H = H; dp.M = M; dp.N = N;
    dp.kv_rows = M; dp.kv_tiles = (M + decode_kt(D) - 1) / decode_kt(D);
    dp.q_shared = 0; dp.k_shared = gated ? 0 : 1; dp.kv_same = 0;
    dp.interleave = 0;
    dp.q_groups = (N + decode_nw(D) * kQTile - 1) / (decode_nw(D) * kQTile);
    dp.items = BH * dp.q_groups;
    dp.scale_log2 = pr.scale_log2;
    dp.y = y;
    dp.y_row = tok.row; dp.y_h = tok.h; dp.y_b = tok.b;
    dp.tok_heads_inner = tok.h < tok.row ? 1 : 0;
    dp.tok_stats = ex.tok_stats;
    dp.tok_stats_stride = ex.tok_stats_stride;
    dp.dy = ex.dy;
    rc = launch_decode<E>(D, m_k_q, gated ? m_q16_kv : m_qf_kv, m_z16, dp, st);
    if (rc) return rc;
    mark(st);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// ------------------------------------------------------------------ token-sharded stages
//
// The token-sharded (context-parallel) form: every rank runs the split passes
// on its own tokens, reduces its chunks to one triple per latent row, and the
// ranks' triples are merged after an all-gather (physicsnemo issue #2024,
// section 2: latent-sized outputs and log-sum-exp statistics rebuild the
// globally normalised attention; decoding stays local).

// One split pass over this rank's tokens, reduced to one unnormalised triple
// per latent row: O at triple[0, rows*D), (m, l) as float2 at triple + rows*D.
// q is [H,M,D] (q_shared) or [B,H,M,D]; v == k reads each tile once (synthesis).
template <typename E>
int cp_split(const Problem& pr, const Buffers& bu, const void* q, bool q_shared, const void* kk, const void* vv,
             float* triple, cudaStream_t st) {
    const int B = pr.B, H = pr.H, N = pr.N, M = pr.M, D = pr.D, BH = B * H;
    const CUtensorMapDataType ty = Elem<E>::kMapType;
    const bool kv_same = kk == vv;
    CUtensorMap mq, mk, mv;
    bool ok = make_map(&mq, ty, q, M, H, q_shared ? 1 : B, D, contiguous_rows(M, H, D), kQTile) &&
              make_map(&mk, ty, kk, N, H, B, D, pr.tok, split_kt(D)) &&
              make_map(&mv, ty, vv, N, H, B, D, pr.tok, split_kt(D));
    if (!ok) return 3;
    Params sp{};
    sp.mode = kSplit;
    sp.B = B; sp.H = H; sp.M = M; sp.N = N;
    sp.kv_rows = N; sp.kv_tiles = (N + split_kt(D) - 1) / split_kt(D);
    sp.tok_heads_inner = pr.tok.h < pr.tok.row ? 1 : 0;
    sp.q_shared = q_shared ? 1 : 0; sp.k_shared = 0; sp.kv_same = kv_same ? 1 : 0;
    sp.interleave = interleaved(M) ? 1 : 0;
    sp.row_groups = row_groups(M);
    sp.chunks = pr.chunks;
    sp.chunk_tiles = pr.chunk_len / split_kt(D);
    sp.items = BH * pr.chunks * sp.row_groups;
    sp.scale_log2 = pr.scale_log2;
    sp.part_O = bu.part_O;
    sp.part_ml = bu.part_ml;
    int rc = launch_split<E>(D, mq, mk, kv_same ? mk : mv, sp, st);
    if (rc) return rc;
    const int64_t rows = (int64_t)BH * M;
    MergeParams mp{};
    mp.part_O = bu.part_O; mp.part_ml = bu.part_ml; mp.chunks = pr.chunks * parts_per_chunk(M);
    mp.B = B; mp.H = H; mp.M = M;
    mp.mode = kMergeTriple;
    mp.out_f32 = triple;
    mp.out_ml = reinterpret_cast<float2*>(triple + rows * D);
    launch_merge_d<E>(D, mp, rows, st);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// Decode of this rank's tokens against the merged latents: keys q ([H,M,D]
// when q_shared, else the [B,H,M,D] routing queries) and values z [B,H,M,D].
template <typename E>
int cp_decode(const Problem& pr, const void* q, bool q_shared, const void* z16, const void* kk, void* y,
              cudaStream_t st, float2* tok_stats = nullptr, int64_t tok_stats_stride = 0, const void* dy = nullptr) {
    const int B = pr.B, H = pr.H, N = pr.N, M = pr.M, D = pr.D, BH = B * H;
    const CUtensorMapDataType ty = Elem<E>::kMapType;
    CUtensorMap mq, mk, mv;
    bool ok = make_map(&mq, ty, kk, N, H, B, D, pr.tok, kQTile) &&
              make_map(&mk, ty, q, M, H, q_shared ? 1 : B, D, contiguous_rows(M, H, D), decode_kt(D)) &&
              make_map(&mv, ty, z16, M, H, B, D, contiguous_rows(M, H, D), decode_kt(D));
    if (!ok) return 3;
    Params dp{};
    dp.mode = kDecode;
    dp.B = B; dp.H = H; dp.M = M; dp.N = N;
    dp.kv_rows = M; dp.kv_tiles = (M + decode_kt(D) - 1) / decode_kt(D);
    dp.q_shared = 0; dp.k_shared = q_shared ? 1 : 0; dp.kv_same = 0;
    dp.interleave = 0;
    dp.q_groups = (N + decode_nw(D) * kQTile - 1) / (decode_nw(D) * kQTile);
    dp.items = BH * dp.q_groups;
    dp.scale_log2 = pr.scale_log2;
    dp.y = y;
    dp.y_row = pr.tok.row; dp.y_h = pr.tok.h; dp.y_b = pr.tok.b;
    dp.tok_heads_inner = pr.tok.h < pr.tok.row ? 1 : 0;
    dp.tok_stats = tok_stats;
    dp.tok_stats_stride = tok_stats_stride;
    dp.dy = dy;
    int rc = launch_decode<E>(D, mq, mk, mv, dp, st);
    if (rc) return rc;
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

}  // namespace tc
}  // namespace flarepp
