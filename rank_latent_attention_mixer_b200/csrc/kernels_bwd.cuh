// Backward of the FLARE++ mixer (SIMT: fp32 arithmetic on the FMA pipe,
// exponentials on MUFU), for every I/O dtype.
//
// The forward (FLARE.py README, "FLARE++" code block) is three softmax
// attentions O = softmax_rows(scale * A B^T) C:
//     synthesis  q_dyn = SDPA(q0, k0, k0)   rows = latents, columns = tokens
//     encode     z     = SDPA(q, k, v)      rows = latents, columns = tokens
//     decode     y     = SDPA(k, q, z)      rows = tokens,  columns = latents
// with q = q_fixed + gate * q_dyn.  For one attention, with P its row-softmax
// weights, dO the gradient of its output and D_r = <dO_r, O_r> (which equals
// sum_j P_rj <dO_r, C_j>), the chain rule through the softmax gives
//     dS_rj = P_rj (<dO_r, C_j> - D_r)
//     dA_r  = scale sum_j dS_rj B_j      (row side: a sum over columns)
//     dB_j  = scale sum_r dS_rj A_r      (column side: a sum over rows)
//     dC_j  =       sum_r P_rj dO_r      (column side)
// Every sum over the N tokens is split into token chunks, written as fp32
// partials and summed by a reduce kernel (deterministic, no atomics); every
// sum over the M latents is taken inside one thread group that holds the
// latents in shared memory.  P is recomputed from the scores and the row's
// log-sum-exp (log2 units): P = 2^(scale log2(e) <A_r, B_j> - lse_r).
//
// Thread mapping: a row (one token or one latent) belongs to G = max(1, D/32)
// adjacent lanes, each holding DS = D/G of its dimensions in registers; dot
// products are reduced across the G lanes by shuffles.  Shared-memory rows are
// stored with the lanes' float4s interleaved (float4 i of lane g at i*G + g),
// so the G lanes read adjacent words and the other row groups of the warp read
// the same words (broadcast): no bank conflicts.
#pragma once

#include "common.cuh"

namespace flarepp {
namespace bwd {

constexpr int kThreads = 128;

template <int D>
struct Lanes {
    static constexpr int G = D >= 64 ? D / 32 : 1;     // lanes per row
    static constexpr int DS = D / G;                    // dimensions per lane
    static constexpr int F4 = DS / 4;                   // float4s per lane
    static constexpr int ROWS = kThreads / G;           // rows per CTA
    static constexpr int TILE = 4096 / D;               // rows per shared-memory stage (two arrays: 32 KB)
};

template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = 1; o < G; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Copies `cnt` rows of D elements (row r at src + r*stride, 16-byte aligned)
// into shared memory as fp32 in the interleaved layout; all threads of the CTA
// take part.
template <typename T, int D>
__device__ __forceinline__ void stage_rows(float* __restrict__ dst, const T* __restrict__ src, int64_t stride,
                                           int cnt) {
    using L = Lanes<D>;
    constexpr int VEC = 16 / sizeof(T);      // elements per 16-byte load
    constexpr int VPR = D / VEC;             // loads per row
    for (int i = threadIdx.x; i < cnt * VPR; i += kThreads) {
        const int r = i / VPR, c = i % VPR;
        float tmp[VEC];
        load_row_f32<T, VEC>(src + (int64_t)r * stride + c * VEC, tmp);
#pragma unroll
        for (int e = 0; e < VEC / 4; ++e) {
            const int f = c * (VEC / 4) + e;                  // float4 index within the row
            const int slot = (f % L::F4) * L::G + f / L::F4;  // interleaved position
            reinterpret_cast<float4*>(dst)[r * (D / 4) + slot] =
                make_float4(tmp[4 * e], tmp[4 * e + 1], tmp[4 * e + 2], tmp[4 * e + 3]);
        }
    }
}

// This lane's DS dimensions of shared row j.
template <int D>
__device__ __forceinline__ void read_slice(const float* __restrict__ s, int j, int g, float (&out)[Lanes<D>::DS]) {
    using L = Lanes<D>;
#pragma unroll
    for (int i = 0; i < L::F4; ++i) {
        const float4 v = reinterpret_cast<const float4*>(s)[j * (D / 4) + i * L::G + g];
        out[4 * i] = v.x; out[4 * i + 1] = v.y; out[4 * i + 2] = v.z; out[4 * i + 3] = v.w;
    }
}

// This lane's DS dimensions of a global row (lane g holds dims [g*DS, g*DS+DS)).
template <typename T, int D>
__device__ __forceinline__ void load_slice(const T* __restrict__ row, int g, float (&out)[Lanes<D>::DS]) {
    load_row_f32<T, Lanes<D>::DS>(row + g * Lanes<D>::DS, out);
}

template <int N>
__device__ __forceinline__ float dot(const float (&a)[N], const float (&b)[N]) {
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < N; ++d) s = fmaf(a[d], b[d], s);
    return s;
}

struct Params {
    int B, H, N, M;
    int64_t tok_row, tok_h, tok_b;   // element strides of the token tensors (k0, k, v, dy and their gradients)
    float scale_log2;                // softmax scale * log2(e)
    float scale;
    int chunks, chunk_len;           // token chunks of the latent-side kernels
    // latent side ([B,H,M,...] rows of (b, h) start at (b*q_batch_heads + h)*M)
    const void* Qlat;                // the latent operand of the attention (q, q_fixed or q0), type TQ
    int q_batch_heads;               // H for [B,H,M,D], 0 for [H,M,D] shared over the batch
    const float* Zlat;               // decode values z [B,H,M,D]
    const float* dOlat;              // output gradient of a latent-row attention [B,H,M,D]
    const float* lse_lat;            // [B,H,M] log-sum-exp of a latent-row attention (log2 units)
    const float* delta_lat;          // [B,H,M] <dO_m, O_m>
    // token side
    const void* Ktok;                // keys (type T)
    const void* Vtok;                // values (type T; == Ktok for the synthesis)
    const void* dYtok;               // decode output gradient dy (type T)
    float* lse_tok;                  // [B,H,N] decode log-sum-exp per token (log2 units)
    float* delta_tok;                // [B,H,N] <dy_n, y_n>
    float* dk_acc;                   // [B,H,N,D] fp32: the decode's share of dk
    void* dK;                        // outputs in the token layout, type T
    void* dV;
    float* part1;                    // [chunks][B*H][M][D]
    float* part2;
};

// Decode, row side (one token per thread group): recomputes the token's
// softmax over the M latents (log-sum-exp, and y to get <dy, y>), then
// dk_dec = scale sum_m dS_nm q_m.  Writes the token's log-sum-exp and <dy, y>
// for the column side.
template <typename T, typename TQ, int D>
__global__ void __launch_bounds__(kThreads)
decode_rows(Params p) {
    using L = Lanes<D>;
    constexpr int DS = L::DS, G = L::G, MC = L::TILE;
    __shared__ __align__(16) float sQ[MC * D];
    __shared__ __align__(16) float sZ[MC * D];
    pdl_wait();
    const int bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
    const int g = threadIdx.x % G;
    const int n = blockIdx.x * L::ROWS + threadIdx.x / G;
    const bool active = n < p.N;
    const int64_t tok = (int64_t)b * p.tok_b + (int64_t)h * p.tok_h + (int64_t)(active ? n : 0) * p.tok_row;
    float ks[DS], dys[DS], acc[DS];
#pragma unroll
    for (int d = 0; d < DS; ++d) { ks[d] = 0.f; dys[d] = 0.f; acc[d] = 0.f; }
    if (active) {
        load_slice<T, D>(reinterpret_cast<const T*>(p.Ktok) + tok, g, ks);
        load_slice<T, D>(reinterpret_cast<const T*>(p.dYtok) + tok, g, dys);
#pragma unroll
        for (int d = 0; d < DS; ++d) ks[d] *= p.scale_log2;
    }
    const TQ* Qbh = reinterpret_cast<const TQ*>(p.Qlat) + (int64_t)(b * p.q_batch_heads + h) * p.M * D;
    const float* Zbh = p.Zlat + (int64_t)bh * p.M * D;
    const bool one_stage = p.M <= MC;

    // pass 1: online softmax over the latents, y accumulated unnormalised in acc
    float mx = -INFINITY, l = 0.f;
    for (int m0 = 0; m0 < p.M; m0 += MC) {
        const int cnt = min(MC, p.M - m0);
        __syncthreads();
        stage_rows<TQ, D>(sQ, Qbh + (int64_t)m0 * D, D, cnt);
        stage_rows<float, D>(sZ, Zbh + (int64_t)m0 * D, D, cnt);
        __syncthreads();
        for (int j = 0; j < cnt; ++j) {
            float r[DS];
            read_slice<D>(sQ, j, g, r);
            const float t = group_sum<G>(dot(ks, r));
            if (t > mx) {
                const float corr = ex2_mufu(mx - t);
                l *= corr;
#pragma unroll
                for (int d = 0; d < DS; ++d) acc[d] *= corr;
                mx = t;
            }
            const float w = ex2_mufu(t - mx);
            l += w;
            read_slice<D>(sZ, j, g, r);
#pragma unroll
            for (int d = 0; d < DS; ++d) acc[d] = fmaf(w, r[d], acc[d]);
        }
    }
    const float lse = mx + log2f(l);
    const float delta = group_sum<G>(dot(dys, acc)) / l;

    // pass 2: dS and the row-side sum
#pragma unroll
    for (int d = 0; d < DS; ++d) acc[d] = 0.f;
    for (int m0 = 0; m0 < p.M; m0 += MC) {
        const int cnt = min(MC, p.M - m0);
        if (!one_stage) {
            __syncthreads();
            stage_rows<TQ, D>(sQ, Qbh + (int64_t)m0 * D, D, cnt);
            stage_rows<float, D>(sZ, Zbh + (int64_t)m0 * D, D, cnt);
            __syncthreads();
        }
        for (int j = 0; j < cnt; ++j) {
            float qr[DS], zr[DS];
            read_slice<D>(sQ, j, g, qr);
            read_slice<D>(sZ, j, g, zr);
            const float t = group_sum<G>(dot(ks, qr));
            const float dp = group_sum<G>(dot(dys, zr));
            const float ds = ex2_mufu(t - lse) * (dp - delta);
#pragma unroll
            for (int d = 0; d < DS; ++d) acc[d] = fmaf(ds, qr[d], acc[d]);
        }
    }
    pdl_launch_dependents();
    if (active) {
#pragma unroll
        for (int d = 0; d < DS; ++d) acc[d] *= p.scale;
        store_row<float, DS>(p.dk_acc + ((int64_t)bh * p.N + n) * D + g * DS, acc);
        if (g == 0) {
            p.lse_tok[(int64_t)bh * p.N + n] = lse;
            p.delta_tok[(int64_t)bh * p.N + n] = delta;
        }
    }
}

// Decode, column side (one latent per thread group, one token chunk per CTA):
// the chunk's partial sums  dq_dec(m) = sum_n dS_nm k_n  (part1, scale applied
// by the reduce) and  dz(m) = sum_n P_nm dy_n  (part2).
template <typename T, typename TQ, int D>
__global__ void __launch_bounds__(kThreads)
decode_cols(Params p) {
    using L = Lanes<D>;
    constexpr int DS = L::DS, G = L::G, TILE = L::TILE;
    __shared__ __align__(16) float sK[TILE * D];
    __shared__ __align__(16) float sY[TILE * D];
    __shared__ float sL[TILE], sDelta[TILE];
    pdl_wait();
    const int c = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
    const int g = threadIdx.x % G;
    const int m = blockIdx.z * L::ROWS + threadIdx.x / G;
    const bool active = m < p.M;
    float qs[DS], zs[DS], a1[DS], a2[DS];
#pragma unroll
    for (int d = 0; d < DS; ++d) { qs[d] = 0.f; zs[d] = 0.f; a1[d] = 0.f; a2[d] = 0.f; }
    if (active) {
        load_slice<TQ, D>(reinterpret_cast<const TQ*>(p.Qlat) + ((int64_t)(b * p.q_batch_heads + h) * p.M + m) * D,
                          g, qs);
        load_slice<float, D>(p.Zlat + ((int64_t)bh * p.M + m) * D, g, zs);
#pragma unroll
        for (int d = 0; d < DS; ++d) qs[d] *= p.scale_log2;
    }
    const int64_t base = (int64_t)b * p.tok_b + (int64_t)h * p.tok_h;
    const T* Kbh = reinterpret_cast<const T*>(p.Ktok) + base;
    const T* Ybh = reinterpret_cast<const T*>(p.dYtok) + base;
    const int n0 = c * p.chunk_len, n1 = min(p.N, n0 + p.chunk_len);
    for (int t0 = n0; t0 < n1; t0 += TILE) {
        const int cnt = min(TILE, n1 - t0);
        __syncthreads();
        stage_rows<T, D>(sK, Kbh + (int64_t)t0 * p.tok_row, p.tok_row, cnt);
        stage_rows<T, D>(sY, Ybh + (int64_t)t0 * p.tok_row, p.tok_row, cnt);
        for (int i = threadIdx.x; i < cnt; i += kThreads) {
            sL[i] = p.lse_tok[(int64_t)bh * p.N + t0 + i];
            sDelta[i] = p.delta_tok[(int64_t)bh * p.N + t0 + i];
        }
        __syncthreads();
        for (int j = 0; j < cnt; ++j) {
            float kr[DS], yr[DS];
            read_slice<D>(sK, j, g, kr);
            read_slice<D>(sY, j, g, yr);
            const float t = group_sum<G>(dot(qs, kr));
            const float dp = group_sum<G>(dot(zs, yr));
            const float pw = ex2_mufu(t - sL[j]);
            const float ds = pw * (dp - sDelta[j]);
#pragma unroll
            for (int d = 0; d < DS; ++d) {
                a1[d] = fmaf(ds, kr[d], a1[d]);
                a2[d] = fmaf(pw, yr[d], a2[d]);
            }
        }
    }
    pdl_launch_dependents();
    if (active) {
        const int64_t row = ((int64_t)c * p.B * p.H + bh) * p.M + m;
        store_row<float, DS>(p.part1 + row * D + g * DS, a1);
        store_row<float, DS>(p.part2 + row * D + g * DS, a2);
    }
}

// Encode or synthesis, row side (one latent per thread group, one token chunk
// per CTA): the chunk's partial  dq(m) = sum_n dS_mn k_n  (part1; scale applied
// by the reduce), with P_mn = 2^(t_mn - lse_m) and dS_mn = P_mn(<dO_m, v_n> - D_m).
template <typename T, typename TQ, int D>
__global__ void __launch_bounds__(kThreads)
latent_rows(Params p) {
    using L = Lanes<D>;
    constexpr int DS = L::DS, G = L::G, TILE = L::TILE;
    __shared__ __align__(16) float sK[TILE * D];
    __shared__ __align__(16) float sV[TILE * D];
    pdl_wait();
    const int c = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
    const int g = threadIdx.x % G;
    const int m = blockIdx.z * L::ROWS + threadIdx.x / G;
    const bool active = m < p.M;
    const bool same_kv = p.Ktok == p.Vtok;
    float qs[DS], dos[DS], a1[DS];
    float lse = 0.f, delta = 0.f;
#pragma unroll
    for (int d = 0; d < DS; ++d) { qs[d] = 0.f; dos[d] = 0.f; a1[d] = 0.f; }
    if (active) {
        const int64_t lrow = (int64_t)bh * p.M + m;
        load_slice<TQ, D>(reinterpret_cast<const TQ*>(p.Qlat) + ((int64_t)(b * p.q_batch_heads + h) * p.M + m) * D,
                          g, qs);
        load_slice<float, D>(p.dOlat + lrow * D, g, dos);
#pragma unroll
        for (int d = 0; d < DS; ++d) qs[d] *= p.scale_log2;
        lse = p.lse_lat[lrow];
        delta = p.delta_lat[lrow];
    }
    const int64_t base = (int64_t)b * p.tok_b + (int64_t)h * p.tok_h;
    const T* Kbh = reinterpret_cast<const T*>(p.Ktok) + base;
    const T* Vbh = reinterpret_cast<const T*>(p.Vtok) + base;
    const int n0 = c * p.chunk_len, n1 = min(p.N, n0 + p.chunk_len);
    for (int t0 = n0; t0 < n1; t0 += TILE) {
        const int cnt = min(TILE, n1 - t0);
        __syncthreads();
        stage_rows<T, D>(sK, Kbh + (int64_t)t0 * p.tok_row, p.tok_row, cnt);
        if (!same_kv) stage_rows<T, D>(sV, Vbh + (int64_t)t0 * p.tok_row, p.tok_row, cnt);
        __syncthreads();
        const float* sVv = same_kv ? sK : sV;
        for (int j = 0; j < cnt; ++j) {
            float kr[DS], vr[DS];
            read_slice<D>(sK, j, g, kr);
            read_slice<D>(sVv, j, g, vr);
            const float t = group_sum<G>(dot(qs, kr));
            const float dp = group_sum<G>(dot(dos, vr));
            const float ds = ex2_mufu(t - lse) * (dp - delta);
#pragma unroll
            for (int d = 0; d < DS; ++d) a1[d] = fmaf(ds, kr[d], a1[d]);
        }
    }
    pdl_launch_dependents();
    if (active) {
        const int64_t row = ((int64_t)c * p.B * p.H + bh) * p.M + m;
        store_row<float, DS>(p.part1 + row * D + g * DS, a1);
    }
}

// Encode or synthesis, column side (one token per thread group, all M latents
// through shared memory): dk_n = scale sum_m dS_mn q_m and dv_n = sum_m P_mn dO_m.
// Encode: dK = dk + the decode's share (dk_acc), dV = dv.  Synthesis (keys
// and values are both k0): dK = dk + dv, dV unused.
template <typename T, typename TQ, int D>
__global__ void __launch_bounds__(kThreads)
token_cols(Params p) {
    using L = Lanes<D>;
    constexpr int DS = L::DS, G = L::G, MC = L::TILE;
    __shared__ __align__(16) float sQ[MC * D];
    __shared__ __align__(16) float sO[MC * D];
    __shared__ float sL[MC], sDelta[MC];
    pdl_wait();
    const int bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
    const int g = threadIdx.x % G;
    const int n = blockIdx.x * L::ROWS + threadIdx.x / G;
    const bool active = n < p.N;
    const bool same_kv = p.Ktok == p.Vtok;
    const int64_t tok = (int64_t)b * p.tok_b + (int64_t)h * p.tok_h + (int64_t)(active ? n : 0) * p.tok_row;
    float ks[DS], vs[DS], ak[DS], av[DS];
#pragma unroll
    for (int d = 0; d < DS; ++d) { ks[d] = 0.f; vs[d] = 0.f; ak[d] = 0.f; av[d] = 0.f; }
    if (active) {
        load_slice<T, D>(reinterpret_cast<const T*>(p.Ktok) + tok, g, vs);
#pragma unroll
        for (int d = 0; d < DS; ++d) ks[d] = vs[d] * p.scale_log2;
        if (!same_kv) load_slice<T, D>(reinterpret_cast<const T*>(p.Vtok) + tok, g, vs);
    }
    const TQ* Qbh = reinterpret_cast<const TQ*>(p.Qlat) + (int64_t)(b * p.q_batch_heads + h) * p.M * D;
    const float* Obh = p.dOlat + (int64_t)bh * p.M * D;
    for (int m0 = 0; m0 < p.M; m0 += MC) {
        const int cnt = min(MC, p.M - m0);
        __syncthreads();
        stage_rows<TQ, D>(sQ, Qbh + (int64_t)m0 * D, D, cnt);
        stage_rows<float, D>(sO, Obh + (int64_t)m0 * D, D, cnt);
        for (int i = threadIdx.x; i < cnt; i += kThreads) {
            sL[i] = p.lse_lat[(int64_t)bh * p.M + m0 + i];
            sDelta[i] = p.delta_lat[(int64_t)bh * p.M + m0 + i];
        }
        __syncthreads();
        for (int j = 0; j < cnt; ++j) {
            float qr[DS], orow[DS];
            read_slice<D>(sQ, j, g, qr);
            read_slice<D>(sO, j, g, orow);
            const float t = group_sum<G>(dot(ks, qr));
            const float dp = group_sum<G>(dot(vs, orow));
            const float pw = ex2_mufu(t - sL[j]);
            const float ds = pw * (dp - sDelta[j]);
#pragma unroll
            for (int d = 0; d < DS; ++d) {
                ak[d] = fmaf(ds, qr[d], ak[d]);
                av[d] = fmaf(pw, orow[d], av[d]);
            }
        }
    }
    pdl_launch_dependents();
    if (active) {
        if (same_kv) {
#pragma unroll
            for (int d = 0; d < DS; ++d) ak[d] = fmaf(p.scale, ak[d], av[d]);
        } else {
            float prev[DS];
            load_row_f32<float, DS>(p.dk_acc + ((int64_t)bh * p.N + n) * D + g * DS, prev);
#pragma unroll
            for (int d = 0; d < DS; ++d) ak[d] = fmaf(p.scale, ak[d], prev[d]);
            store_row<T, DS>(reinterpret_cast<T*>(p.dV) + tok + g * DS, av);
        }
        store_row<T, DS>(reinterpret_cast<T*>(p.dK) + tok + g * DS, ak);
    }
}

// Sums of the token-chunk partials, one warp per latent row (b, h, m); lane
// i holds dims i, i+32, ... (D/32 of them, or one for lanes < D when D < 32).
enum ReduceMode {
    kReduceDecode = 0,      // dz = sum part2; dq = scale sum part1; D_enc = <dz, z>
    kReduceEncode = 1,      // dq += scale sum part1; gated: dq_dyn = gate dq, D_syn = <dq_dyn, q_dyn>
    kReduceSynthesis = 2    // dq0_b = scale sum part1
};

struct ReduceParams {
    const float* part1;
    const float* part2;
    int chunks;
    int B, H, M;
    float scale;
    int mode;
    const float* z;         // decode: z [B,H,M,D]
    float* dz;              // decode: out
    float* dq;              // decode: out; encode: in/out
    float* delta;           // decode: D_enc; encode (gated): D_syn
    const float* gate;      // encode: gate [H] (NULL: closed gate)
    const float* qdyn;      // encode (gated): q_dyn [B,H,M,D]
    float* dqdyn;           // encode (gated): out
    float* dq0b;            // synthesis: out [B,H,M,D]
    // tensor-core backward only (else NULL): the 16-bit copy of dz (decode) or dq_dyn
    // (encode), and the next pass's (log-sum-exp, Delta) per latent row at
    // stats_out[(b*H + h)*stats_stride + m], the log-sum-exp read from lse_in[row]
    void* out16;
    float2* stats_out;
    int64_t stats_stride;
    const float* lse_in;
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
reduce_partials(ReduceParams p) {
    constexpr int PL = D >= 32 ? D / 32 : 1;    // dims per lane
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)p.B * p.H * p.M;
    const int64_t row = (int64_t)blockIdx.x * 8 + warp;
    if (row >= rows) return;
    const bool lane_on = D >= 32 || lane < D;
    const int64_t cstride = rows * D;
    float s1[PL], s2[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) { s1[i] = 0.f; s2[i] = 0.f; }
    if (lane_on) {
        for (int c = 0; c < p.chunks; ++c) {
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int64_t idx = c * cstride + row * D + lane + 32 * i;
                s1[i] += p.part1[idx];
                if (p.mode == kReduceDecode) s2[i] += p.part2[idx];
            }
        }
    }
    float dsum = 0.f;
    if (p.mode == kReduceDecode) {
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            if (!lane_on) continue;
            const int64_t idx = row * D + lane + 32 * i;
            p.dz[idx] = s2[i];
            if constexpr (sizeof(T) == 2) {
                if (p.out16) static_cast<T*>(p.out16)[idx] = from_f32<T>(s2[i]);
            }
            p.dq[idx] = p.scale * s1[i];
            dsum = fmaf(s2[i], p.z[idx], dsum);
        }
    } else if (p.mode == kReduceEncode) {
        const int h = (int)((row / p.M) % p.H);
        const float gh = p.gate ? p.gate[h] : 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            if (!lane_on) continue;
            const int64_t idx = row * D + lane + 32 * i;
            const float dq = fmaf(p.scale, s1[i], p.dq[idx]);
            p.dq[idx] = dq;
            if (p.gate) {
                const float dd = gh * dq;
                p.dqdyn[idx] = dd;
                if constexpr (sizeof(T) == 2) {
                    if (p.out16) static_cast<T*>(p.out16)[idx] = from_f32<T>(dd);
                }
                dsum = fmaf(dd, p.qdyn[idx], dsum);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < PL; ++i)
            if (lane_on) p.dq0b[row * D + lane + 32 * i] = p.scale * s1[i];
    }
    pdl_launch_dependents();
    if (p.mode == kReduceDecode || (p.mode == kReduceEncode && p.gate)) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        if (lane == 0) {
            p.delta[row] = dsum;
            if (p.stats_out)
                p.stats_out[(row / p.M) * p.stats_stride + row % p.M] = make_float2(p.lse_in[row], dsum);
        }
    }
}

// Gradient through the head-wise RMS normalisation of the synthesis seeds and
// keys/values (physicsnemo issue #2024, FLARE++ list, "Normalizing the
// synthesis call"; read as xh = x r, r = (mean_d x^2 + eps)^(-1/2)): for each
// row x and the gradient g of its normalised form, dx = r (g - xh <g, xh> / D)
// (chain rule, dr/dx_j = -r^3 x_j / D), written over g.  One thread per row,
// 32 dimensions at a time in two passes (sums, then the update); HBM-bound:
// x read once (twice from cache), g read and written.
template <typename TX, typename TG, int D>
__global__ void __launch_bounds__(256)
rms_backward_rows(const TX* __restrict__ x, TG* __restrict__ g, int64_t rows, float eps) {
    constexpr int C = D < 32 ? D : 32;
    pdl_wait();
    pdl_launch_dependents();
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const TX* xr = x + r * D;
    TG* gr = g + r * D;
    float ss = 0.f, gx = 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += C) {
        float xv[C], gv[C];
        load_row_f32<TX, C>(xr + c0, xv);
        load_row_f32<TG, C>(gr + c0, gv);
#pragma unroll
        for (int i = 0; i < C; ++i) {
            ss = fmaf(xv[i], xv[i], ss);
            gx = fmaf(gv[i], xv[i], gx);
        }
    }
    const float rs = rsqrtf(ss * (1.f / D) + eps);
    const float coef = rs * rs * gx * (1.f / D);        // <g, xh> / D divided by r: xh_i = x_i r
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += C) {
        float xv[C], gv[C];
        load_row_f32<TX, C>(xr + c0, xv);
        load_row_f32<TG, C>(gr + c0, gv);
#pragma unroll
        for (int i = 0; i < C; ++i) gv[i] = rs * fmaf(-xv[i], coef, gv[i]);
        store_row<TG, C>(gr + c0, gv);
    }
}

// The same step when x and g have one type (the token rows: k0 and dk0): one
// 16-byte chunk per lane, the lanes of a row combining their sums by shuffles,
// so every warp access is coalesced (one read of x, one read and one write of
// g).  A grid-stride loop over rows.
template <typename T, int D>
__global__ void __launch_bounds__(256)
rms_backward_rows_coop(const T* __restrict__ x, T* __restrict__ g, int64_t rows, float eps) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int E = 16 / sizeof(T);              // elements per chunk
    constexpr int C = D / E;                       // chunks per row (<= 32)
    constexpr int RW = 32 / C;                     // rows per warp pass
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t first = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    for (int64_t r0 = first * RW; r0 < rows; r0 += warps * RW) {
        const int64_t r = r0 + lane / C;
        const bool in = r < rows;                  // every lane still takes part in the shuffles
        const int64_t off = r * D + (lane % C) * E;
        float xv[E], gv[E];
        float ss = 0.f, gx = 0.f;
        if (in) {
            load_row_f32<T, E>(x + off, xv);
            load_row_f32<T, E>(g + off, gv);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                ss = fmaf(xv[e], xv[e], ss);
                gx = fmaf(gv[e], xv[e], gx);
            }
        }
#pragma unroll
        for (int o = C / 2; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            gx += __shfl_xor_sync(0xffffffffu, gx, o);
        }
        if (in) {
            const float rs = rsqrtf(ss * (1.f / D) + eps);
            const float coef = rs * rs * gx * (1.f / D);
#pragma unroll
            for (int e = 0; e < E; ++e) gv[e] = rs * fmaf(-xv[e], coef, gv[e]);
            store_row<T, E>(g + off, gv);
        }
    }
}

// fp32 rows -> the 16-bit I/O type (round to nearest even): the tensor-core
// operands q and z rebuilt from a saved forward state, the same rounding the
// forward's merge applies.  n is a multiple of 8 (whole rows of D >= 16).
template <typename E>
__global__ void __launch_bounds__(256)
round_to_io(const float* __restrict__ in, E* __restrict__ out, int64_t n) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * 8;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n; i += stride) {
        float v[8];
        load_row_f32<float, 8>(in + i, v);
        store_row<E, 8>(out + i, v);
    }
}

// Per token, <dy_n, y_n> into the second member of the backward's per-token
// statistics (the first, the decode's log-sum-exp, came from the forward):
// tok_stats[(b*H + h)*stride + n].y.  y and dy in the I/O type E, token rows
// addressed by their strides; one 16-byte chunk per lane, the lanes of a row
// combining by shuffles (coalesced; HBM-bound: one read of dy and of y).
template <typename E, int D>
__global__ void __launch_bounds__(256)
token_delta(float2* __restrict__ tok_stats, int64_t stride, const E* __restrict__ dy, const E* __restrict__ y,
            int H, int N, int64_t rows, int64_t tok_row, int64_t tok_h, int64_t tok_b) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int EL = 16 / sizeof(E);             // elements per chunk
    constexpr int C = D / EL;                      // chunks per row (<= 32)
    constexpr int RW = 32 / C;                     // rows per warp pass
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t first = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    for (int64_t r0 = first * RW; r0 < rows; r0 += warps * RW) {
        const int64_t r = r0 + lane / C;           // row = (b*H + h)*N + n
        const bool in = r < rows;
        float sum = 0.f;
        int64_t bh = 0, n = 0;
        if (in) {
            bh = r / N;
            n = r - bh * N;
            const int64_t b = bh / H, h = bh - b * H;
            const int64_t off = b * tok_b + h * tok_h + n * tok_row + (lane % C) * EL;
            float gv[EL], yv[EL];
            load_row_f32<E, EL>(dy + off, gv);
            load_row_f32<E, EL>(y + off, yv);
#pragma unroll
            for (int e = 0; e < EL; ++e) sum = fmaf(gv[e], yv[e], sum);
        }
#pragma unroll
        for (int o = C / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (in && lane % C == 0) tok_stats[bh * stride + n].y = sum;
    }
}

// Gradients of the batch-shared inputs, one CTA per head: dq_fixed[h] =
// sum_b dq[b,h], dq0[h] = sum_b dq0_b[b,h] and dgate[h] = sum_{b,m} <dq, q_dyn>
// (q = q_fixed + gate q_dyn).  Deterministic: fixed summation order.
struct BatchParams {
    int B, H, M;
    const float* dq;        // [B,H,M,D]
    const float* dq0b;      // [B,H,M,D] (gated) or NULL
    const float* qdyn;      // [B,H,M,D] (gated) or NULL
    float* dq_fixed;        // [H,M,D]
    float* dq0;             // [H,M,D] (gated) or NULL
    float* dgate;           // [H] (gated) or NULL
};

template <int D>
__global__ void __launch_bounds__(256)
reduce_batch(BatchParams p) {
    __shared__ float red[256];
    pdl_wait();
    const int h = blockIdx.x;
    const int64_t per_h = (int64_t)p.M * D;
    float gsum = 0.f;
    for (int64_t i = threadIdx.x; i < per_h; i += blockDim.x) {
        float a = 0.f, c = 0.f;
        for (int b = 0; b < p.B; ++b) {
            const int64_t idx = ((int64_t)b * p.H + h) * per_h + i;
            const float dq = p.dq[idx];
            a += dq;
            if (p.dq0b) c += p.dq0b[idx];
            if (p.qdyn) gsum = fmaf(dq, p.qdyn[idx], gsum);
        }
        p.dq_fixed[(int64_t)h * per_h + i] = a;
        if (p.dq0) p.dq0[(int64_t)h * per_h + i] = c;
    }
    if (!p.dgate) return;
    red[threadIdx.x] = gsum;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) p.dgate[h] = red[0];
}

}  // namespace bwd
}  // namespace flarepp
