// SIMT (FFMA, fp32) kernels of the FLARE++ mixer: the split-N partial pass used
// by the synthesis and encode calls, the merge of the partial softmax triples,
// and the decode.  They serve every fp32-I/O call (fp32 products keep the
// 1e-4 accuracy that TF32 tensor-core products would not) and every shape the
// tcgen05 kernels do not cover.
//
// Notation (FLARE.py README, "FLARE++" code block): for one (b, h) the score of
// latent m and token n is S[m, n] = scale * <q[m], k[n]>.  The synthesis and
// encode calls softmax S along n (per latent); the decode softmaxes the same
// kind of score along m (per token).  All exponentials are taken base 2 on
// scores pre-multiplied by scale*log2(e), which is the same softmax.
#pragma once

#include "common.cuh"

namespace flarepp {

constexpr int kSimtThreads = 128;

// Lanes per row of the SIMT kernels: one, or two at D = 128, where a row's
// query and accumulator (2 x 128 floats) would not fit one thread's
// registers; each lane of a pair then holds D/2 of them and the pair sums its
// halves of every score with one shuffle.  The split pass keeps 128 latent
// rows per CTA (128 or 256 threads), so each staged key/value tile serves as
// many rows; the decode keeps 128 threads (64 token rows per CTA at D = 128:
// measured 16.4 ms against 18.7 with 128 rows on 256 threads, 262144 tokens,
// H = 8, M = 256).
constexpr int simt_lanes_per_row(int D) { return D > 64 ? 2 : 1; }
constexpr int simt_split_threads(int D) { return kSimtThreads * simt_lanes_per_row(D); }
constexpr int simt_decode_rows(int D) { return kSimtThreads / simt_lanes_per_row(D); }

// Split-N partial pass: for one (b, h), one chunk of tokens and one block of
// latent rows, the online-softmax triple of every row over the chunk:
// running max (log2 units), sum of weights, and the unnormalised weighted sum
// of the value rows.  Chunks of the same (b, h) are combined by merge_partials;
// this split of the token axis and the log-sum-exp merge is exact up to
// rounding (physicsnemo issue #2024, section 2: the token-sharded encoder
// rebuilds the globally normalised attention from latent-sized outputs and
// log-sum-exp statistics).
struct SplitParams {
    const void* Q;       // latent query rows; (b, h) rows start at row (b*q_batch_heads + h)*M
    int q_batch_heads;   // H when Q is [B,H,M,D]; 0 when Q is [H,M,D] (shared over b)
    const void* K;       // token keys: row n of (b, h) at b*tok_b + h*tok_h + n*tok_row elements
    const void* V;       // token values, same strides (may equal K: synthesis reads k0 twice)
    int64_t tok_row, tok_h, tok_b;
    float* part_O;       // [C][B*H][M][D]
    float2* part_ml;     // [C][B*H][M]: (max in log2 units, sum of weights)
    int B, H, N, M;
    int chunks, chunk_len;
    float scale_log2;    // softmax scale * log2(e)
};

template <int D> struct SimtTile { static constexpr int tokens = 2048 / D; };

template <typename TQ, typename TKV, int D>
__global__ void __launch_bounds__(simt_split_threads(D))
split_partial_simt(SplitParams p) {
    constexpr int TILE = SimtTile<D>::tokens;
    __shared__ __align__(16) float sK[TILE * D];
    __shared__ __align__(16) float sV[TILE * D];

    constexpr int TPR = simt_lanes_per_row(D);
    constexpr int DL = D / TPR;                    // columns of q and O held by this lane
    const int c = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh - b * p.H;
    const int m = blockIdx.z * kSimtThreads + threadIdx.x / TPR;
    const int part = threadIdx.x % TPR;
    const unsigned pair = (TPR == 2 ? 3u : 1u) << ((threadIdx.x & 31) & ~(TPR - 1));
    const bool active = m < p.M;                   // the same for both lanes of a row
    const int n0 = c * p.chunk_len;
    const int n1 = min(p.N, n0 + p.chunk_len);
    const bool same_kv = p.K == p.V;

    float q[DL];
#pragma unroll
    for (int d = 0; d < DL; ++d) q[d] = 0.f;
    if (active) {
        const TQ* qrow = reinterpret_cast<const TQ*>(p.Q) +
                         ((int64_t)(b * p.q_batch_heads + h) * p.M + m) * D + part * DL;
        load_row_f32<TQ, DL>(qrow, q);
#pragma unroll
        for (int d = 0; d < DL; ++d) q[d] *= p.scale_log2;
    }
    float mx = -INFINITY, l = 0.f, acc[DL];
#pragma unroll
    for (int d = 0; d < DL; ++d) acc[d] = 0.f;

    const int64_t base = (int64_t)b * p.tok_b + (int64_t)h * p.tok_h;
    const TKV* Kbh = reinterpret_cast<const TKV*>(p.K) + base;
    const TKV* Vbh = reinterpret_cast<const TKV*>(p.V) + base;
    constexpr int VEC = 16 / sizeof(TKV);          // elements per 16-byte load
    constexpr int VPR = D / VEC;                   // 16-byte loads per row
    for (int t0 = n0; t0 < n1; t0 += TILE) {
        const int cnt = min(TILE, n1 - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < cnt * VPR; i += simt_split_threads(D)) {
            float tmp[VEC];
            const int64_t off = (int64_t)(t0 + i / VPR) * p.tok_row + (i % VPR) * VEC;
            load_row_f32<TKV, VEC>(Kbh + off, tmp);
#pragma unroll
            for (int e = 0; e < VEC; ++e) sK[i * VEC + e] = tmp[e];
            if (!same_kv) {
                load_row_f32<TKV, VEC>(Vbh + off, tmp);
#pragma unroll
                for (int e = 0; e < VEC; ++e) sV[i * VEC + e] = tmp[e];
            }
        }
        __syncthreads();
        const float* sVv = same_kv ? sK : sV;
        if (active) {
            for (int j = 0; j < cnt; ++j) {
                const float* kr = sK + j * D + part * DL;
                float s = 0.f;
#pragma unroll
                for (int d = 0; d < DL; ++d) s = fmaf(q[d], kr[d], s);
                if constexpr (TPR == 2) s += __shfl_xor_sync(pair, s, 1);
                if (s > mx) {
                    const float corr = ex2_mufu(mx - s);
                    l *= corr;
#pragma unroll
                    for (int d = 0; d < DL; ++d) acc[d] *= corr;
                    mx = s;
                }
                const float w = ex2_mufu(s - mx);
                l += w;
                const float* vr = sVv + j * D + part * DL;
#pragma unroll
                for (int d = 0; d < DL; ++d) acc[d] = fmaf(w, vr[d], acc[d]);
            }
        }
    }
    if (active) {
        const int64_t row = ((int64_t)c * p.B * p.H + bh) * p.M + m;
        if (part == 0) p.part_ml[row] = make_float2(mx, l);
        store_row<float, DL>(p.part_O + row * D + part * DL, acc);
    }
}

// Head-wise RMS normalisation of rows of D elements (the synthesis seeds q0
// and keys/values k0; physicsnemo issue #2024, FLARE++ list, "Normalizing the
// synthesis call"): out = x / sqrt(mean_d x^2 + eps), computed in fp32 and
// rounded to T.  Any tensor whose rows of D elements are contiguous in memory
// -- [H,M,D], [B,H,N,D] or [B,N,H,D] -- is `rows` such rows back to back.
// One 16-byte chunk per lane; a row's lanes combine their sums by shuffles.
// HBM-bound: one read and one write of each tensor.  One launch serves two
// tensors: rows [0, rows1) of x1 -> out1, then rows2 rows of x2 -> out2.
template <typename T, int D>
__global__ void __launch_bounds__(256)
rms_normalise_rows(const T* __restrict__ x1, T* __restrict__ out1, int64_t rows1, const T* __restrict__ x2,
                   T* __restrict__ out2, int64_t rows2, float eps) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t rows = rows1 + rows2;
    constexpr int E = 16 / sizeof(T);              // elements per chunk
    constexpr int C = D / E;                       // chunks per row (<= 32)
    constexpr int RW = 32 / C;                     // rows per warp pass
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t first = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    for (int64_t r0 = first * RW; r0 < rows; r0 += warps * RW) {
        const int64_t r = r0 + lane / C;
        const bool in = r < rows;                  // every lane still takes part in the shuffles
        const bool second = r >= rows1;
        const T* src = second ? x2 + (r - rows1) * D : x1 + r * D;
        T* dst = second ? out2 + (r - rows1) * D : out1 + r * D;
        float v[E];
        float ss = 0.f;
        if (in) {
            load_row_f32<T, E>(src + (lane % C) * E, v);
#pragma unroll
            for (int e = 0; e < E; ++e) ss = fmaf(v[e], v[e], ss);
        }
#pragma unroll
        for (int o = C / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (in) {
            const float inv = rsqrtf(ss * (1.f / D) + eps);
#pragma unroll
            for (int e = 0; e < E; ++e) v[e] *= inv;
            store_row<T, E>(dst + (lane % C) * E, v);
        }
    }
}

// Merge of the per-chunk triples of one latent row (one warp per row):
// out = sum_c 2^(m_c - m*) O_c / sum_c 2^(m_c - m*) l_c with m* = max_c m_c.
// Synthesis epilogue: q = q_fixed + gate[h] * out (FLARE.py README, FLARE++
// block, second line).  Encode epilogue: z = out.  Triple mode writes the
// combined triple itself (m*, L = sum_c 2^(m_c - m*) l_c, sum_c 2^(m_c - m*)
// O_c) unnormalised: the local step of the token-sharded form, whose triples
// are merged again across ranks.
enum MergeMode { kMergeSynthesis = 0, kMergeEncode = 1, kMergeTriple = 2 };

// Optional extra outputs of a forward call, kept for its backward: the
// log-sum-exp (log2 units, of the scaled scores) of every latent row of the
// synthesis and encode softmaxes, the synthesis output before the gate, and
// whether to run the decode at all (the backward recomputes it per token).
struct FwdExtras {
    float* lse_syn = nullptr;    // [B,H,M]
    float* lse_enc = nullptr;    // [B,H,M]
    float* qdyn = nullptr;       // [B,H,M,D] fp32
    bool decode = true;
    // tcgen05 decode only: per token (log-sum-exp, <dy, y>) at [(b*H + h)*stride + n];
    // y may then be NULL (not written)
    float2* tok_stats = nullptr;
    int64_t tok_stats_stride = 0;
    const void* dy = nullptr;
};

struct MergeParams {
    const float* part_O;        // part c's O row r at part_O + c*o_part_stride + r*D
    const float2* part_ml;      // part c's (m, l) of row r at part_ml[c*ml_part_stride + r]
    int64_t o_part_stride;      // floats; 0 = B*H*M*D (parts stored back to back)
    int64_t ml_part_stride;     // float2s; 0 = B*H*M
    float2* out_ml;             // triple mode: combined (m*, L) per row
    int chunks;
    int B, H, M;
    int mode;                   // MergeMode
    const void* q_fixed;        // [H,M,D] in the I/O dtype (synthesis epilogue, or copied to q_copy_out)
    const float* gate;          // [H] (synthesis epilogue)
    float* out_f32;             // [B,H,M,D]
    void* out_16;               // [B,H,M,D] in the I/O dtype (16-bit I/O only; may be null)
    float* user_out;            // optional [B,H,M,D]
    float* q_copy_out;          // optional: closed gate, write q = q_fixed broadcast over b
    float* lse_out;             // optional [B,H,M]: m* + log2(L), the row's log-sum-exp in log2 units
    float* pregate_out;         // optional [B,H,M,D] (synthesis): the merged value before the gate
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
merge_partials(MergeParams p) {
    // A warp merges one latent row.  Each lane loads one float4 of a chunk's O
    // row, so LPC = D/4 lanes cover a chunk and the warp takes CPI = 32/LPC
    // chunks per iteration (D = 128: one chunk in four float4s per lane).
    constexpr int V4 = D / 4;
    constexpr int LPC = V4 < 32 ? V4 : 32;
    constexpr int CPI = 32 / LPC;
    constexpr int F4PL = V4 / LPC;              // float4s per lane per chunk
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)p.B * p.H * p.M;
    const int64_t row = (int64_t)blockIdx.x * 8 + warp;
    if (row >= rows) return;
    const int m = (int)(row % p.M);
    const int h = (int)((row / p.M) % p.H);
    const int64_t ostride = p.o_part_stride ? p.o_part_stride : rows * D;
    const int64_t mlstride = p.ml_part_stride ? p.ml_part_stride : rows;

    float mstar = -INFINITY;
    for (int c = lane; c < p.chunks; c += 32) mstar = fmaxf(mstar, p.part_ml[c * mlstride + row].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));

    const int sub = lane / LPC, li = lane % LPC;
    float L = 0.f;
    float4 acc[F4PL];
#pragma unroll
    for (int i = 0; i < F4PL; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < p.chunks; c0 += CPI) {
        const int c = c0 + sub;
        if (c < p.chunks) {
            const float2 ml = p.part_ml[c * mlstride + row];
            const float4* o4 = reinterpret_cast<const float4*>(p.part_O + c * ostride + row * D);
            const float w = ml.y > 0.f ? ex2_mufu(ml.x - mstar) : 0.f;   // empty chunk contributes nothing
            L = fmaf(w, ml.y, L);
#pragma unroll
            for (int i = 0; i < F4PL; ++i) {
                const float4 v = o4[li + LPC * i];
                acc[i].x = fmaf(w, v.x, acc[i].x); acc[i].y = fmaf(w, v.y, acc[i].y);
                acc[i].z = fmaf(w, v.z, acc[i].z); acc[i].w = fmaf(w, v.w, acc[i].w);
            }
        }
    }
    // combine the CPI chunk groups of the warp (lanes li, li + LPC, ...)
#pragma unroll
    for (int o = 16; o >= LPC; o >>= 1) {
        L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
        for (int i = 0; i < F4PL; ++i) {
            acc[i].x += __shfl_xor_sync(0xffffffffu, acc[i].x, o);
            acc[i].y += __shfl_xor_sync(0xffffffffu, acc[i].y, o);
            acc[i].z += __shfl_xor_sync(0xffffffffu, acc[i].z, o);
            acc[i].w += __shfl_xor_sync(0xffffffffu, acc[i].w, o);
        }
    }
    if (sub != 0) return;
    if (p.lse_out && li == 0) p.lse_out[row] = mstar + log2f(L);
    if (p.mode == kMergeTriple) {
#pragma unroll
        for (int i = 0; i < F4PL; ++i)
            reinterpret_cast<float4*>(p.out_f32 + row * D)[li + LPC * i] = acc[i];
        if (li == 0) p.out_ml[row] = make_float2(mstar, L);
        return;
    }
    const float inv = 1.f / L;
    const T* qf = reinterpret_cast<const T*>(p.q_fixed) + ((int64_t)h * p.M + m) * D;
#pragma unroll
    for (int i = 0; i < F4PL; ++i) {
        const int d0 = 4 * (li + LPC * i);
        float val[4] = {acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = d0 + e;
            if (p.pregate_out) p.pregate_out[row * D + d] = val[e];
            if (p.mode == kMergeSynthesis) val[e] = fmaf(p.gate[h], val[e], to_f32<T>(qf[d]));
            p.out_f32[row * D + d] = val[e];
            if constexpr (sizeof(T) == 2) {
                if (p.out_16) reinterpret_cast<T*>(p.out_16)[row * D + d] = from_f32<T>(val[e]);
            }
            if (p.user_out) p.user_out[row * D + d] = val[e];
            if (p.q_copy_out) p.q_copy_out[row * D + d] = to_f32<T>(qf[d]);
        }
    }
}

// Decode (FLARE.py README, FLARE++ block, last line: y = SDPA(k, q, z)): one
// thread per token; the token's key row is the query, the M latent rows of q
// are the keys and those of z the values.  Latent rows are staged through
// shared memory in chunks of 2048/D rows and every thread reads the same row
// (broadcast); the softmax over M is online across the chunks.
struct DecodeParams {
    const void* Ktok;     // token keys: row n of (b, h) at b*tok_b + h*tok_h + n*tok_row elements
    const void* Qlat;     // latent keys; (b, h) rows start at row (b*q_batch_heads + h)*M
    int q_batch_heads;
    const float* Z;       // [B,H,M,D] fp32
    void* Y;              // output rows, same strides as Ktok
    int64_t tok_row, tok_h, tok_b;
    int B, H, N, M;
    float scale_log2;
};

template <typename T, typename TQ, int D>
__global__ void __launch_bounds__(kSimtThreads)
decode_simt(DecodeParams p) {
    constexpr int MC = 2048 / D;
    __shared__ __align__(16) float sQ[MC * D];
    __shared__ __align__(16) float sZ[MC * D];
    constexpr int TPR = simt_lanes_per_row(D);
    constexpr int DL = D / TPR;                    // columns of the token row held by this lane
    const int bh = blockIdx.y;
    const int b = bh / p.H, h = bh - b * p.H;
    const int n = blockIdx.x * simt_decode_rows(D) + threadIdx.x / TPR;
    const int part = threadIdx.x % TPR;
    const unsigned pair = (TPR == 2 ? 3u : 1u) << ((threadIdx.x & 31) & ~(TPR - 1));
    const bool active = n < p.N;                   // the same for both lanes of a row

    float kq[DL];
#pragma unroll
    for (int d = 0; d < DL; ++d) kq[d] = 0.f;
    if (active) {
        load_row_f32<T, DL>(reinterpret_cast<const T*>(p.Ktok) + (int64_t)b * p.tok_b + (int64_t)h * p.tok_h +
                                (int64_t)n * p.tok_row + part * DL, kq);
#pragma unroll
        for (int d = 0; d < DL; ++d) kq[d] *= p.scale_log2;
    }
    float mx = -INFINITY, l = 0.f, acc[DL];
#pragma unroll
    for (int d = 0; d < DL; ++d) acc[d] = 0.f;

    const TQ* Qbh = reinterpret_cast<const TQ*>(p.Qlat) + (int64_t)(b * p.q_batch_heads + h) * p.M * D;
    const float* Zbh = p.Z + (int64_t)bh * p.M * D;
    constexpr int VEC = 16 / sizeof(TQ);
    for (int m0 = 0; m0 < p.M; m0 += MC) {
        const int cnt = min(MC, p.M - m0);
        __syncthreads();
        for (int i = threadIdx.x; i < cnt * D / VEC; i += kSimtThreads) {
            float tmp[VEC];
            load_row_f32<TQ, VEC>(Qbh + (int64_t)m0 * D + i * VEC, tmp);
#pragma unroll
            for (int e = 0; e < VEC; ++e) sQ[i * VEC + e] = tmp[e];
        }
        for (int i = threadIdx.x; i < cnt * D / 4; i += kSimtThreads)
            reinterpret_cast<float4*>(sZ)[i] = reinterpret_cast<const float4*>(Zbh + (int64_t)m0 * D)[i];
        __syncthreads();
        if (active) {
            for (int j = 0; j < cnt; ++j) {
                const float* qr = sQ + j * D + part * DL;
                float s = 0.f;
#pragma unroll
                for (int d = 0; d < DL; ++d) s = fmaf(kq[d], qr[d], s);
                if constexpr (TPR == 2) s += __shfl_xor_sync(pair, s, 1);
                if (s > mx) {
                    const float corr = ex2_mufu(mx - s);
                    l *= corr;
#pragma unroll
                    for (int d = 0; d < DL; ++d) acc[d] *= corr;
                    mx = s;
                }
                const float w = ex2_mufu(s - mx);
                l += w;
                const float* zr = sZ + j * D + part * DL;
#pragma unroll
                for (int d = 0; d < DL; ++d) acc[d] = fmaf(w, zr[d], acc[d]);
            }
        }
    }
    if (active) {
        const float inv = 1.f / l;
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[d] *= inv;
        store_row<T, DL>(reinterpret_cast<T*>(p.Y) + (int64_t)b * p.tok_b + (int64_t)h * p.tok_h +
                             (int64_t)n * p.tok_row + part * DL, acc);
    }
}

}  // namespace flarepp
