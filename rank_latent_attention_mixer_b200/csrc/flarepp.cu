// C ABI of the FLARE++ mixer forward: argument checks, planning, workspace
// and the launch sequence.  The operation and the ABI contract are documented
// in include/flarepp.h.
//
// Launch sequence for one call (gate open):
//   1. split partial   Q = q0 [H,M,D],  K = V = k0     (synthesis, V = K)
//   2. merge           q = q_fixed + gate * q_dyn       -> q fp32 + I/O dtype
//   3. split partial   Q = q,           K = k, V = v    (encode)
//   4. merge           z                                -> z fp32 + I/O dtype
//   5. decode          y = SDPA(k, q, z)
// With the gate closed, steps 1-2 are skipped and q_fixed is used as q.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/flarepp.h"
#include "common.cuh"
#include "kernels_bwd.cuh"
#include "kernels_bwd_tc.cuh"
#include "kernels_simt.cuh"
#include "kernels_tc.cuh"

namespace flarepp {

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Shape {
    int B, H, N, M, D, dtype;
    int64_t bh() const { return (int64_t)B * H; }
    size_t elem() const { return dtype == FLAREPP_F32 ? 4 : 2; }
    size_t tok_bytes() const { return (size_t)B * H * (size_t)N * D * elem(); }
    size_t lat_bytes() const { return (size_t)H * M * D * elem(); }
};

// Work split and scratch layout of one call.
struct Plan {
    int path;            // flarepp_path_t (SIMT or TCGEN05)
    int chunks;          // token chunks per (b, h) in the split passes
    int chunk_len;       // tokens per chunk
    int row_blocks;      // latent-row blocks per (b, h, chunk) (SIMT)
    float scale_log2;
    tc::RowStrides tok;  // element strides of the token tensors k0, k, v, y (flarepp_layout_t)
    int norm_synthesis;  // RMS-normalise q0 and k0 rows in the synthesis pass
    // byte offsets into the workspace
    size_t off_part_O, off_part_ml, off_q32, off_q16, off_z32, off_z16, off_q0n, off_k0n, total;
};

int check_shape(const Shape& s) {
    if (s.B < 1 || s.H < 1 || s.N < 1 || s.M < 1) return FLAREPP_ERR_INVALID_ARG;
    if (s.dtype != FLAREPP_F32 && s.dtype != FLAREPP_BF16 && s.dtype != FLAREPP_F16) return FLAREPP_ERR_INVALID_ARG;
    if (s.bh() > 65535 || s.M > 4096) return FLAREPP_ERR_UNSUPPORTED;
    if (s.D != 16 && s.D != 32 && s.D != 64 && s.D != 128) return FLAREPP_ERR_UNSUPPORTED;
    return FLAREPP_OK;
}

int tile_tokens_simt(int D) { return 2048 / D; }

bool tc_supported(const Shape& s) { return tc::supported(s.dtype != FLAREPP_F32, s.D, s.M); }

int choose_path(const Shape& s, int requested) {
    if (requested == FLAREPP_PATH_SIMT) return FLAREPP_PATH_SIMT;
    if (requested == FLAREPP_PATH_TCGEN05) return tc_supported(s) ? FLAREPP_PATH_TCGEN05 : -1;
    if (requested != FLAREPP_PATH_AUTO) return -1;
    return tc_supported(s) ? FLAREPP_PATH_TCGEN05 : FLAREPP_PATH_SIMT;
}

int make_plan(const Shape& s, const flarepp_options_t* o, Plan* pl) {
    int rc = check_shape(s);
    if (rc) return rc;
    const int requested = o ? o->path : FLAREPP_PATH_AUTO;
    const int path = choose_path(s, requested);
    if (path < 0) return requested == FLAREPP_PATH_TCGEN05 ? FLAREPP_ERR_UNSUPPORTED : FLAREPP_ERR_INVALID_ARG;
    if (o && o->n_stage_events < 0) return FLAREPP_ERR_INVALID_ARG;
    if (o && o->n_stage_events > 0 && !o->stage_events) return FLAREPP_ERR_INVALID_ARG;
    if (o && o->force_chunks < 0) return FLAREPP_ERR_INVALID_ARG;
    const int layout = o ? o->layout : FLAREPP_LAYOUT_BHND;
    if (o && o->norm_synthesis != 0 && o->norm_synthesis != 1) return FLAREPP_ERR_INVALID_ARG;
    pl->norm_synthesis = o ? o->norm_synthesis : 0;
    if (layout != FLAREPP_LAYOUT_BHND && layout != FLAREPP_LAYOUT_BNHD) return FLAREPP_ERR_INVALID_ARG;
    pl->tok = layout == FLAREPP_LAYOUT_BNHD
                  ? tc::RowStrides{(int64_t)s.H * s.D, s.D, (int64_t)s.N * s.H * s.D}
                  : tc::contiguous_rows(s.N, s.H, s.D);
    pl->path = path;
    const float scale = (o && o->scale > 0.f) ? o->scale : 1.f / std::sqrt((float)s.D);
    if (!std::isfinite(scale)) return FLAREPP_ERR_INVALID_ARG;
    pl->scale_log2 = scale * kLog2e;

    int tile, units_per_bh;
    if (path == FLAREPP_PATH_SIMT) {
        tile = tile_tokens_simt(s.D);
        pl->row_blocks = (s.M + kSimtThreads - 1) / kSimtThreads;
        units_per_bh = pl->row_blocks;
    } else {
        tile = tc::kv_tile(s.D);
        pl->row_blocks = tc::row_groups(s.M);
        units_per_bh = pl->row_blocks;
    }
    const int64_t tiles = (s.N + tile - 1) / tile;
    int64_t chunks;
    if (o && o->force_chunks > 0) {
        chunks = std::min<int64_t>(o->force_chunks, tiles);
    } else if (path == FLAREPP_PATH_SIMT) {
        // Enough CTAs for several waves over the SMs, but chunks of >= 1 tile.
        const int64_t target = 4 * kNumSMs;
        chunks = (target + s.bh() * units_per_bh - 1) / (s.bh() * units_per_bh);
        chunks = std::max<int64_t>(1, std::min<int64_t>(chunks, tiles));
    } else {
        chunks = tc::choose_chunks(s.bh() * units_per_bh, tiles, kNumSMs,
                                   tc::interleaved(s.M) ? tc::kSplitNW : 1);
    }
    int64_t tiles_per_chunk = (tiles + chunks - 1) / chunks;
    pl->chunk_len = (int)std::min<int64_t>(tiles_per_chunk * tile, INT32_MAX);
    pl->chunks = (int)((s.N + (int64_t)pl->chunk_len - 1) / pl->chunk_len);
    const int parts = path == FLAREPP_PATH_SIMT ? pl->chunks : pl->chunks * tc::parts_per_chunk(s.M);

    const size_t rows = (size_t)s.bh() * s.M;
    size_t off = 0;
    pl->off_part_O = off;  off = align_up(off + (size_t)parts * rows * s.D * sizeof(float));
    pl->off_part_ml = off; off = align_up(off + (size_t)parts * rows * sizeof(float2));
    pl->off_q32 = off;     off = align_up(off + rows * s.D * sizeof(float));
    pl->off_q16 = off;     off = align_up(off + rows * s.D * sizeof(uint16_t));     // q in the 16-bit I/O dtype
    pl->off_z32 = off;     off = align_up(off + rows * s.D * sizeof(float));
    pl->off_z16 = off;     off = align_up(off + rows * s.D * sizeof(uint16_t));
    // the normalised synthesis seeds and keys/values (norm_synthesis)
    pl->off_q0n = off;     off = align_up(off + (pl->norm_synthesis ? s.lat_bytes() : 0));
    pl->off_k0n = off;     off = align_up(off + (pl->norm_synthesis ? s.tok_bytes() : 0));
    pl->total = off;
    return FLAREPP_OK;
}

// Caller-provided events recorded around the launches (flarepp_options_t).
struct StageEvents {
    void* const* ev = nullptr;
    int n = 0;
    int next = 0;
    void mark(cudaStream_t st) {
        if (next < n && ev[next]) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[next]), st);
        ++next;
    }
};

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int check_pointers(const Shape& s, const void* q0, const void* q_fixed, const float* gate,
                   const void* k0, const void* k, const void* v, const void* y) {
    const bool gated = gate != nullptr;
    if (!q_fixed || !k || !v || !y) return FLAREPP_ERR_INVALID_ARG;
    if (gated && (!q0 || !k0)) return FLAREPP_ERR_INVALID_ARG;
    const void* tensors[] = {q_fixed, k, v, y, gated ? q0 : nullptr, gated ? k0 : nullptr};
    for (const void* t : tensors)
        if (t && !aligned16(t)) return FLAREPP_ERR_INVALID_ARG;
    if (gated && (reinterpret_cast<uintptr_t>(gate) & 3u)) return FLAREPP_ERR_INVALID_ARG;
    const size_t tb = s.tok_bytes(), lb = s.lat_bytes();
    if (overlaps(y, tb, k, tb) || overlaps(y, tb, v, tb) || overlaps(y, tb, q_fixed, lb)) return FLAREPP_ERR_INVALID_ARG;
    if (gated && (overlaps(y, tb, k0, tb) || overlaps(y, tb, q0, lb) ||
                  overlaps(y, tb, gate, (size_t)s.H * sizeof(float))))
        return FLAREPP_ERR_INVALID_ARG;
    return FLAREPP_OK;
}

template <typename T>
int run_simt(const Shape& s, const Plan& pl, const void* q0, const void* q_fixed, const float* gate,
             const void* k0, const void* k, const void* v, void* y, char* ws,
             float* q_out, float* z_out, StageEvents& ev, cudaStream_t st, const FwdExtras& ex) {
    const bool gated = gate != nullptr;
    float* part_O = reinterpret_cast<float*>(ws + pl.off_part_O);
    float2* part_ml = reinterpret_cast<float2*>(ws + pl.off_part_ml);
    float* q32 = reinterpret_cast<float*>(ws + pl.off_q32);
    void* q16 = ws + pl.off_q16;
    float* z32 = reinterpret_cast<float*>(ws + pl.off_z32);
    void* z16 = ws + pl.off_z16;

    const dim3 split_grid(pl.chunks, (unsigned)s.bh(), pl.row_blocks);
    const int64_t rows = s.bh() * s.M;
    const dim3 merge_grid((unsigned)((rows + 7) / 8));
    const dim3 dec_grid((unsigned)((s.N + simt_decode_rows(s.D) - 1) / simt_decode_rows(s.D)), (unsigned)s.bh());

    SplitParams sp{};
    sp.tok_row = pl.tok.row; sp.tok_h = pl.tok.h; sp.tok_b = pl.tok.b;
    sp.part_O = part_O; sp.part_ml = part_ml;
    sp.B = s.B; sp.H = s.H; sp.N = s.N; sp.M = s.M;
    sp.chunks = pl.chunks; sp.chunk_len = pl.chunk_len; sp.scale_log2 = pl.scale_log2;
    MergeParams mp{};
    mp.part_O = part_O; mp.part_ml = part_ml; mp.chunks = pl.chunks;
    mp.B = s.B; mp.H = s.H; mp.M = s.M; mp.q_fixed = q_fixed; mp.gate = gate;
    DecodeParams dp{};
    dp.Ktok = k; dp.Z = z32; dp.Y = y; dp.B = s.B; dp.H = s.H; dp.N = s.N; dp.M = s.M;
    dp.tok_row = pl.tok.row; dp.tok_h = pl.tok.h; dp.tok_b = pl.tok.b;
    dp.scale_log2 = pl.scale_log2;

#define FLAREPP_SIMT_DISPATCH(DD)                                                                  \
    case DD: {                                                                                     \
        ev.mark(st);                                                                               \
        if (gated) {                                                                               \
            sp.Q = q0; sp.q_batch_heads = 0; sp.K = k0; sp.V = k0;                                 \
            split_partial_simt<T, T, DD><<<split_grid, simt_split_threads(DD), 0, st>>>(sp);                 \
            ev.mark(st);                                                                           \
            mp.mode = kMergeSynthesis; mp.out_f32 = q32; mp.out_16 = q16; mp.user_out = q_out;   \
            mp.q_copy_out = nullptr; mp.lse_out = ex.lse_syn; mp.pregate_out = ex.qdyn;           \
            merge_partials<T, DD><<<merge_grid, 256, 0, st>>>(mp);                                 \
            ev.mark(st);                                                                           \
            sp.Q = q32; sp.q_batch_heads = s.H; sp.K = k; sp.V = v;                                \
            split_partial_simt<float, T, DD><<<split_grid, simt_split_threads(DD), 0, st>>>(sp);             \
            ev.mark(st);                                                                           \
        } else {                                                                                   \
            sp.Q = q_fixed; sp.q_batch_heads = 0; sp.K = k; sp.V = v;                              \
            split_partial_simt<T, T, DD><<<split_grid, simt_split_threads(DD), 0, st>>>(sp);                 \
            ev.mark(st);                                                                           \
        }                                                                                          \
        mp.mode = kMergeEncode; mp.out_f32 = z32; mp.out_16 = z16; mp.user_out = z_out;          \
        mp.q_copy_out = gated ? nullptr : q_out; mp.lse_out = ex.lse_enc; mp.pregate_out = nullptr; \
        merge_partials<T, DD><<<merge_grid, 256, 0, st>>>(mp);                                     \
        ev.mark(st);                                                                               \
        if (!ex.decode) {                                                                          \
        } else if (gated) {                                                                        \
            dp.Qlat = q32; dp.q_batch_heads = s.H;                                                 \
            decode_simt<T, float, DD><<<dec_grid, kSimtThreads, 0, st>>>(dp);                      \
            ev.mark(st);                                                                           \
        } else {                                                                                   \
            dp.Qlat = q_fixed; dp.q_batch_heads = 0;                                               \
            decode_simt<T, T, DD><<<dec_grid, kSimtThreads, 0, st>>>(dp);                          \
            ev.mark(st);                                                                           \
        }                                                                                          \
        break;                                                                                     \
    }
    switch (s.D) {
        FLAREPP_SIMT_DISPATCH(16)
        FLAREPP_SIMT_DISPATCH(32)
        FLAREPP_SIMT_DISPATCH(64)
        FLAREPP_SIMT_DISPATCH(128)
        default: return FLAREPP_ERR_UNSUPPORTED;
    }
#undef FLAREPP_SIMT_DISPATCH
    (void)q16; (void)z16;
    return cudaGetLastError() == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
}

int run(const Shape& s, const Plan& pl, const void* q0, const void* q_fixed, const float* gate,
        const void* k0, const void* k, const void* v, void* y, char* ws,
        float* q_out, float* z_out, StageEvents& ev, cudaStream_t st, const FwdExtras& ex = FwdExtras{}) {
    if (pl.path == FLAREPP_PATH_TCGEN05) {
        tc::Buffers bu{};
        bu.part_O = reinterpret_cast<float*>(ws + pl.off_part_O);
        bu.part_ml = reinterpret_cast<float2*>(ws + pl.off_part_ml);
        bu.q32 = reinterpret_cast<float*>(ws + pl.off_q32);
        bu.q16 = ws + pl.off_q16;
        bu.z32 = reinterpret_cast<float*>(ws + pl.off_z32);
        bu.z16 = ws + pl.off_z16;
        tc::Problem pr{};
        pr.B = s.B; pr.H = s.H; pr.N = s.N; pr.M = s.M; pr.D = s.D;
        pr.tok = pl.tok;
        pr.chunks = pl.chunks; pr.chunk_len = pl.chunk_len; pr.scale_log2 = pl.scale_log2;
        auto mark = [&ev](cudaStream_t t) { ev.mark(t); };
        if (s.dtype == FLAREPP_F16)
            return tc::run<__half>(pr, bu, q0, q_fixed, gate, k0, k, v, y, q_out, z_out, mark, st, ex);
        return tc::run<__nv_bfloat16>(pr, bu, q0, q_fixed, gate, k0, k, v, y, q_out, z_out, mark, st, ex);
    }
    if (s.dtype == FLAREPP_F32)
        return run_simt<float>(s, pl, q0, q_fixed, gate, k0, k, v, y, ws, q_out, z_out, ev, st, ex);
    if (s.dtype == FLAREPP_F16)
        return run_simt<__half>(s, pl, q0, q_fixed, gate, k0, k, v, y, ws, q_out, z_out, ev, st, ex);
    return run_simt<__nv_bfloat16>(s, pl, q0, q_fixed, gate, k0, k, v, y, ws, q_out, z_out, ev, st, ex);
}

// Head-wise RMS normalisation of the synthesis seeds (H*M rows) and
// keys/values (B*H*N rows) into their workspace copies, one launch.
constexpr float kNormEps = 1e-6f;

template <typename T>
void launch_rms_norm(const Shape& s, const void* q0, void* q0n, const void* k0, void* k0n, cudaStream_t st) {
    const int64_t rows1 = (int64_t)s.H * s.M, rows2 = s.bh() * s.N;
    const int rw = 32 / (s.D * (int)sizeof(T) / 16);                // rows per warp pass
    const int64_t want = (rows1 + rows2 + 8 * rw - 1) / (8 * rw);
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)kNumSMs * 16);
    const T* a = static_cast<const T*>(q0);
    const T* b = static_cast<const T*>(k0);
    T* oa = static_cast<T*>(q0n);
    T* ob = static_cast<T*>(k0n);
    switch (s.D) {
        case 16: rms_normalise_rows<T, 16><<<grid, 256, 0, st>>>(a, oa, rows1, b, ob, rows2, kNormEps); break;
        case 32: rms_normalise_rows<T, 32><<<grid, 256, 0, st>>>(a, oa, rows1, b, ob, rows2, kNormEps); break;
        case 64: rms_normalise_rows<T, 64><<<grid, 256, 0, st>>>(a, oa, rows1, b, ob, rows2, kNormEps); break;
        default: rms_normalise_rows<T, 128><<<grid, 256, 0, st>>>(a, oa, rows1, b, ob, rows2, kNormEps); break;
    }
}

void rms_norm(const Shape& s, const void* q0, void* q0n, const void* k0, void* k0n, cudaStream_t st) {
    if (s.dtype == FLAREPP_F32) launch_rms_norm<float>(s, q0, q0n, k0, k0n, st);
    else if (s.dtype == FLAREPP_F16) launch_rms_norm<__half>(s, q0, q0n, k0, k0n, st);
    else launch_rms_norm<__nv_bfloat16>(s, q0, q0n, k0, k0n, st);
}

// Caller-registered scratch per device (flarepp_set_workspace), used by the
// forward entries that receive no workspace in their options.
constexpr int kMaxDevices = 64;
struct RegisteredWorkspace {
    void* ptr = nullptr;
    size_t bytes = 0;
};
std::mutex g_registered_mu;
RegisteredWorkspace g_registered[kMaxDevices];

// The current device's registered scratch if it holds at least `need` bytes.
char* registered_workspace(size_t need) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_registered_mu);
    const RegisteredWorkspace& r = g_registered[dev];
    return r.ptr && r.bytes >= need ? static_cast<char*>(r.ptr) : nullptr;
}

int forward(const void* q0, const void* q_fixed, const float* gate, const void* k0, const void* k,
            const void* v, void* y, int B, int H, int N, int M, int D, int dtype,
            const flarepp_options_t* opts, void* stream, const FwdExtras& ex = FwdExtras{}) {
    const Shape s{B, H, N, M, D, dtype};
    Plan pl{};
    int rc = make_plan(s, opts, &pl);
    if (rc) return rc;
    rc = check_pointers(s, q0, q_fixed, gate, k0, k, v, y);
    if (rc) return rc;
    float* q_out = opts ? opts->q_out : nullptr;
    float* z_out = opts ? opts->z_out : nullptr;
    if ((q_out && !aligned16(q_out)) || (z_out && !aligned16(z_out))) return FLAREPP_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* ws = nullptr;
    bool owned = false;
    if (opts && opts->workspace) {
        if (opts->workspace_bytes < pl.total) return FLAREPP_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(opts->workspace) % kAlign) return FLAREPP_ERR_INVALID_ARG;
        ws = static_cast<char*>(opts->workspace);
    } else if ((ws = registered_workspace(pl.total)) == nullptr) {
        if (cudaMallocAsync(reinterpret_cast<void**>(&ws), pl.total, st) != cudaSuccess) {
            cudaGetLastError();
            return FLAREPP_ERR_WORKSPACE;
        }
        owned = true;
    }
    StageEvents ev;
    if (opts && opts->n_stage_events > 0) {
        ev.ev = opts->stage_events;
        ev.n = opts->n_stage_events;
    }
    if (pl.norm_synthesis && gate) {
        // the synthesis reads normalised copies (its own stage for the events)
        ev.mark(st);
        rms_norm(s, q0, ws + pl.off_q0n, k0, ws + pl.off_k0n, st);
        q0 = ws + pl.off_q0n;
        k0 = ws + pl.off_k0n;
    }
    rc = run(s, pl, q0, q_fixed, gate, k0, k, v, y, ws, q_out, z_out, ev, st, ex);
    if (owned && cudaFreeAsync(ws, st) != cudaSuccess && rc == FLAREPP_OK) rc = FLAREPP_ERR_CUDA;
    return rc;
}

// ------------------------------------------------------------------ fixed device scratch
//
// Scratch for flarepp_mixer_fwd_noalloc: a file-scope device array, so that
// entry point never allocates.  Every GPU that loads this library holds the
// array until the process exits.  All calls share it; each call overwrites the
// part it uses, and nothing in it needs to start at zero (every byte a kernel
// reads was written earlier in the same call).  Two such calls whose kernels
// overlap on the GPU race on it.
constexpr size_t kStaticScratchBytes = FLAREPP_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is asked from the
// runtime once per device, with that device current, and cached.
void* static_scratch_address() {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

// Largest token-chunk count whose scratch fits the fixed array (0: none fits).
int chunks_fitting_static_scratch(const Shape& s) {
    Plan pl{};
    if (make_plan(s, nullptr, &pl)) return 0;
    if (pl.total <= kStaticScratchBytes) return pl.chunks;
    int lo = 1, hi = pl.chunks, best = 0;
    while (lo <= hi) {
        const int mid = lo + (hi - lo) / 2;
        flarepp_options_t o{};
        o.force_chunks = mid;
        Plan q{};
        if (make_plan(s, &o, &q)) return 0;
        if (q.total <= kStaticScratchBytes) {
            best = mid;
            lo = mid + 1;
        } else {
            hi = mid - 1;
        }
    }
    return best;
}

// ------------------------------------------------------------------ host-buffer entry
//
// The (b, h) slices of the mixer are independent problems, so the host entry
// streams them: the copy-in of slice i+1 (stream `in`), the forward of slice
// i (the caller's stream) and the copy-out of slice i-1 (stream `out`) overlap,
// with two device slots for a slice's inputs and output.  Staging comes from
// a library-owned memory pool that keeps its memory reserved between calls,
// so repeated calls do not map and unmap device memory.
struct HostResources {
    cudaStream_t in = nullptr, out = nullptr;
    cudaMemPool_t pool = nullptr;
    bool ready = false;
};

HostResources* host_resources() {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static HostResources res[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    HostResources& r = res[dev];
    if (!r.ready) {
        cudaMemPoolProps props{};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        if ((!r.in && cudaStreamCreateWithFlags(&r.in, cudaStreamNonBlocking) != cudaSuccess) ||
            (!r.out && cudaStreamCreateWithFlags(&r.out, cudaStreamNonBlocking) != cudaSuccess) ||
            (!r.pool && cudaMemPoolCreate(&r.pool, &props) != cudaSuccess)) {
            cudaGetLastError();
            return nullptr;
        }
        uint64_t keep = UINT64_MAX;
        if (cudaMemPoolSetAttribute(r.pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        r.ready = true;
    }
    return &r;
}

int host_forward(const void* q0, const void* q_fixed, const float* gate, const void* k0, const void* k,
                 const void* v, void* y, int B, int H, int N, int M, int D, int dtype, void* stream) {
    const Shape s{B, H, N, M, D, dtype};
    Plan pl{};
    int rc = make_plan(s, nullptr, &pl);
    if (rc) return rc;
    const bool gated = gate != nullptr;
    if (!q_fixed || !k || !v || !y || (gated && (!q0 || !k0))) return FLAREPP_ERR_INVALID_ARG;
    const Shape s1{1, 1, N, M, D, dtype};
    Plan p1{};
    rc = make_plan(s1, nullptr, &p1);
    if (rc) return rc;
    HostResources* hr = host_resources();
    if (!hr) return FLAREPP_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    const size_t t1 = (size_t)N * D * s.elem(), l1 = (size_t)M * D * s.elem();
    const int slices = B * H;
    // device layout: latent inputs of all heads, then two slots of
    // [k0 (gated), k, v, y, scratch] for one (b, h) slice each
    size_t off = 0;
    const size_t o_qf = off; off = align_up(off + (size_t)H * l1);
    const size_t o_q0 = off; if (gated) off = align_up(off + (size_t)H * l1);
    const size_t o_g = off;  if (gated) off = align_up(off + (size_t)H * sizeof(float));
    size_t o_slot[2], o_k0 = 0, o_k, o_v, o_y, o_ws;
    {
        size_t so = 0;
        o_k0 = so; if (gated) so = align_up(so + t1);
        o_k = so;  so = align_up(so + t1);
        o_v = so;  so = align_up(so + t1);
        o_y = so;  so = align_up(so + t1);
        o_ws = so; so = align_up(so + p1.total);
        o_slot[0] = off; off += so;
        o_slot[1] = off; off += so;
    }
    char* d = nullptr;
    if (cudaMallocFromPoolAsync(reinterpret_cast<void**>(&d), off, hr->pool, st) != cudaSuccess) {
        cudaGetLastError();
        return FLAREPP_ERR_WORKSPACE;
    }
    cudaEvent_t ev_lat = nullptr, in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
    bool ok = cudaEventCreateWithFlags(&ev_lat, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < 2 && ok; ++i)
        ok = cudaEventCreateWithFlags(&in_done[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&out_done[i], cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(d + o_qf, q_fixed, (size_t)H * l1, cudaMemcpyHostToDevice, st) == cudaSuccess;
    if (ok && gated)
        ok = cudaMemcpyAsync(d + o_q0, q0, (size_t)H * l1, cudaMemcpyHostToDevice, st) == cudaSuccess &&
             cudaMemcpyAsync(d + o_g, gate, (size_t)H * sizeof(float), cudaMemcpyHostToDevice, st) == cudaSuccess;
    // the copy streams may touch the block only after its stream-ordered allocation
    ok = ok && cudaEventRecord(ev_lat, st) == cudaSuccess && cudaStreamWaitEvent(hr->in, ev_lat, 0) == cudaSuccess &&
         cudaStreamWaitEvent(hr->out, ev_lat, 0) == cudaSuccess;
    rc = ok ? FLAREPP_OK : FLAREPP_ERR_CUDA;
    const char* hk0 = static_cast<const char*>(k0);
    const char* hk = static_cast<const char*>(k);
    const char* hv = static_cast<const char*>(v);
    char* hy = static_cast<char*>(y);
    for (int si = 0; si < slices && rc == FLAREPP_OK; ++si) {
        const int slot = si & 1, h = si % H;
        char* base = d + o_slot[slot];
        const size_t ho = (size_t)si * t1;
        ok = si < 2 || cudaStreamWaitEvent(hr->in, comp_done[slot], 0) == cudaSuccess;   // slot inputs consumed
        if (ok && gated) ok = cudaMemcpyAsync(base + o_k0, hk0 + ho, t1, cudaMemcpyHostToDevice, hr->in) == cudaSuccess;
        ok = ok && cudaMemcpyAsync(base + o_k, hk + ho, t1, cudaMemcpyHostToDevice, hr->in) == cudaSuccess &&
             cudaMemcpyAsync(base + o_v, hv + ho, t1, cudaMemcpyHostToDevice, hr->in) == cudaSuccess &&
             cudaEventRecord(in_done[slot], hr->in) == cudaSuccess &&
             cudaStreamWaitEvent(st, in_done[slot], 0) == cudaSuccess &&
             (si < 2 || cudaStreamWaitEvent(st, out_done[slot], 0) == cudaSuccess);        // slot output drained
        if (!ok) { rc = FLAREPP_ERR_CUDA; break; }
        flarepp_options_t o{};
        o.workspace = base + o_ws;
        o.workspace_bytes = p1.total;
        rc = forward(gated ? d + o_q0 + (size_t)h * l1 : nullptr, d + o_qf + (size_t)h * l1,
                     gated ? reinterpret_cast<float*>(d + o_g) + h : nullptr, gated ? base + o_k0 : nullptr,
                     base + o_k, base + o_v, base + o_y, 1, 1, N, M, D, dtype, &o, stream);
        if (rc) break;
        ok = cudaEventRecord(comp_done[slot], st) == cudaSuccess &&
             cudaStreamWaitEvent(hr->out, comp_done[slot], 0) == cudaSuccess &&
             cudaMemcpyAsync(hy + ho, base + o_y, t1, cudaMemcpyDeviceToHost, hr->out) == cudaSuccess &&
             cudaEventRecord(out_done[slot], hr->out) == cudaSuccess;
        if (!ok) rc = FLAREPP_ERR_CUDA;
    }
    // join the copy streams back into the caller's stream, release, synchronise
    for (int i = 0; i < 2; ++i) {
        if (in_done[i] && cudaStreamWaitEvent(st, in_done[i], 0) != cudaSuccess && rc == FLAREPP_OK) rc = FLAREPP_ERR_CUDA;
        if (out_done[i] && cudaStreamWaitEvent(st, out_done[i], 0) != cudaSuccess && rc == FLAREPP_OK) rc = FLAREPP_ERR_CUDA;
    }
    if (cudaFreeAsync(d, st) != cudaSuccess && rc == FLAREPP_OK) rc = FLAREPP_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess && rc == FLAREPP_OK) rc = FLAREPP_ERR_CUDA;
    cudaEvent_t evs[] = {ev_lat, in_done[0], in_done[1], comp_done[0], comp_done[1], out_done[0], out_done[1]};
    for (cudaEvent_t e : evs)
        if (e) cudaEventDestroy(e);
    return rc;
}

// ------------------------------------------------------------------ token-sharded stages
//
// A latent state (the routing queries q or the latents z after the merge
// across ranks) is [B,H,M,D] fp32 followed, for 16-bit I/O, by the same rows
// in the I/O dtype (the tensor-core operand) at latent_16_offset().

size_t latent_16_offset(const Shape& s) { return align_up((size_t)s.bh() * s.M * s.D * sizeof(float)); }

size_t latent_state_bytes(const Shape& s) {
    return latent_16_offset(s) + (s.dtype == FLAREPP_F32 ? 0 : (size_t)s.bh() * s.M * s.D * 2);
}

// Workspace of one staged call: the caller's, or stream-ordered from the pool.
struct StageScratch {
    char* ws = nullptr;
    bool owned = false;
    cudaStream_t st = nullptr;
    int acquire(const Plan& pl, const flarepp_options_t* opts, cudaStream_t stream) {
        st = stream;
        if (opts && opts->workspace) {
            if (opts->workspace_bytes < pl.total) return FLAREPP_ERR_WORKSPACE;
            if (reinterpret_cast<uintptr_t>(opts->workspace) % kAlign) return FLAREPP_ERR_INVALID_ARG;
            ws = static_cast<char*>(opts->workspace);
            return FLAREPP_OK;
        }
        if (cudaMallocAsync(reinterpret_cast<void**>(&ws), pl.total, st) != cudaSuccess) {
            cudaGetLastError();
            return FLAREPP_ERR_WORKSPACE;
        }
        owned = true;
        return FLAREPP_OK;
    }
    int release(int rc) {
        if (owned && cudaFreeAsync(ws, st) != cudaSuccess && rc == FLAREPP_OK) rc = FLAREPP_ERR_CUDA;
        owned = false;
        return rc;
    }
};

template <typename T>
void simt_triple(const Shape& s, const Plan& pl, char* ws, float* triple, cudaStream_t st) {
    const int64_t rows = s.bh() * s.M;
    MergeParams mp{};
    mp.part_O = reinterpret_cast<float*>(ws + pl.off_part_O);
    mp.part_ml = reinterpret_cast<float2*>(ws + pl.off_part_ml);
    mp.chunks = pl.chunks;
    mp.B = s.B; mp.H = s.H; mp.M = s.M;
    mp.mode = kMergeTriple;
    mp.out_f32 = triple;
    mp.out_ml = reinterpret_cast<float2*>(triple + rows * s.D);
    const dim3 grid((unsigned)((rows + 7) / 8));
    switch (s.D) {
        case 16: merge_partials<T, 16><<<grid, 256, 0, st>>>(mp); break;
        case 32: merge_partials<T, 32><<<grid, 256, 0, st>>>(mp); break;
        case 64: merge_partials<T, 64><<<grid, 256, 0, st>>>(mp); break;
        default: merge_partials<T, 128><<<grid, 256, 0, st>>>(mp); break;
    }
}

// SIMT split pass + local reduction.  The query rows are the I/O dtype T when
// shared ([H,M,D]) and the fp32 part of a latent state otherwise.
template <typename T>
int simt_cp_partials(const Shape& s, const Plan& pl, const void* q, bool q_shared, const void* k, const void* v,
                     float* triple, char* ws, cudaStream_t st) {
    SplitParams sp{};
    sp.Q = q; sp.q_batch_heads = q_shared ? 0 : s.H; sp.K = k; sp.V = v;
    sp.tok_row = pl.tok.row; sp.tok_h = pl.tok.h; sp.tok_b = pl.tok.b;
    sp.part_O = reinterpret_cast<float*>(ws + pl.off_part_O);
    sp.part_ml = reinterpret_cast<float2*>(ws + pl.off_part_ml);
    sp.B = s.B; sp.H = s.H; sp.N = s.N; sp.M = s.M;
    sp.chunks = pl.chunks; sp.chunk_len = pl.chunk_len; sp.scale_log2 = pl.scale_log2;
    const dim3 grid(pl.chunks, (unsigned)s.bh(), pl.row_blocks);
#define FLAREPP_CP_SPLIT(DD)                                                                       \
    case DD:                                                                                       \
        if (q_shared) split_partial_simt<T, T, DD><<<grid, simt_split_threads(DD), 0, st>>>(sp);             \
        else split_partial_simt<float, T, DD><<<grid, simt_split_threads(DD), 0, st>>>(sp);                  \
        break;
    switch (s.D) {
        FLAREPP_CP_SPLIT(16)
        FLAREPP_CP_SPLIT(32)
        FLAREPP_CP_SPLIT(64)
        FLAREPP_CP_SPLIT(128)
        default: return FLAREPP_ERR_UNSUPPORTED;
    }
#undef FLAREPP_CP_SPLIT
    simt_triple<T>(s, pl, ws, triple, st);
    return cudaGetLastError() == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
}

template <typename T>
int simt_cp_decode(const Shape& s, const Plan& pl, const void* q, bool q_shared, const float* z32, const void* k,
                   void* y, cudaStream_t st) {
    DecodeParams dp{};
    dp.Ktok = k; dp.Qlat = q; dp.q_batch_heads = q_shared ? 0 : s.H; dp.Z = z32; dp.Y = y;
    dp.B = s.B; dp.H = s.H; dp.N = s.N; dp.M = s.M;
    dp.tok_row = pl.tok.row; dp.tok_h = pl.tok.h; dp.tok_b = pl.tok.b;
    dp.scale_log2 = pl.scale_log2;
    const dim3 grid((unsigned)((s.N + simt_decode_rows(s.D) - 1) / simt_decode_rows(s.D)), (unsigned)s.bh());
#define FLAREPP_CP_DEC(DD)                                                                         \
    case DD:                                                                                       \
        if (q_shared) decode_simt<T, T, DD><<<grid, kSimtThreads, 0, st>>>(dp);                    \
        else decode_simt<T, float, DD><<<grid, kSimtThreads, 0, st>>>(dp);                         \
        break;
    switch (s.D) {
        FLAREPP_CP_DEC(16)
        FLAREPP_CP_DEC(32)
        FLAREPP_CP_DEC(64)
        FLAREPP_CP_DEC(128)
        default: return FLAREPP_ERR_UNSUPPORTED;
    }
#undef FLAREPP_CP_DEC
    return cudaGetLastError() == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
}

tc::Problem tc_problem(const Shape& s, const Plan& pl) {
    tc::Problem pr{};
    pr.B = s.B; pr.H = s.H; pr.N = s.N; pr.M = s.M; pr.D = s.D;
    pr.tok = pl.tok;
    pr.chunks = pl.chunks; pr.chunk_len = pl.chunk_len; pr.scale_log2 = pl.scale_log2;
    return pr;
}

tc::Buffers tc_buffers(const Plan& pl, char* ws) {
    tc::Buffers bu{};
    bu.part_O = reinterpret_cast<float*>(ws + pl.off_part_O);
    bu.part_ml = reinterpret_cast<float2*>(ws + pl.off_part_ml);
    return bu;
}

int cp_partials(const void* q, int q_shared, const void* k, const void* v, float* triple, int B, int H, int N,
                int M, int D, int dtype, const flarepp_options_t* opts, void* stream) {
    const Shape s{B, H, N, M, D, dtype};
    Plan pl{};
    int rc = make_plan(s, opts, &pl);
    if (rc) return rc;
    if (!q || !k || !v || !triple || (q_shared != 0 && q_shared != 1)) return FLAREPP_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(triple)) return FLAREPP_ERR_INVALID_ARG;
    const size_t tb = s.tok_bytes();
    const size_t trb = (size_t)s.bh() * M * (D + 2) * sizeof(float);
    if (overlaps(triple, trb, k, tb) || overlaps(triple, trb, v, tb)) return FLAREPP_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    StageScratch sc;
    rc = sc.acquire(pl, opts, st);
    if (rc) return rc;
    if (pl.norm_synthesis) {
        // normalised copies of this call's seeds and keys/values (the synthesis call)
        if (!q_shared || k != v) {
            return sc.release(FLAREPP_ERR_INVALID_ARG);
        }
        rms_norm(s, q, sc.ws + pl.off_q0n, k, sc.ws + pl.off_k0n, st);
        q = sc.ws + pl.off_q0n;
        k = v = sc.ws + pl.off_k0n;
    }
    // a latent state's operand part: the I/O-dtype copy (tensor cores) or fp32 (SIMT)
    const void* q16 = q_shared ? q : static_cast<const char*>(q) + latent_16_offset(s);
    if (pl.path == FLAREPP_PATH_TCGEN05) {
        const tc::Problem pr = tc_problem(s, pl);
        const tc::Buffers bu = tc_buffers(pl, sc.ws);
        rc = dtype == FLAREPP_F16 ? tc::cp_split<__half>(pr, bu, q16, q_shared, k, v, triple, st)
                                  : tc::cp_split<__nv_bfloat16>(pr, bu, q16, q_shared, k, v, triple, st);
        if (rc) rc = rc == 2 ? FLAREPP_ERR_UNSUPPORTED : FLAREPP_ERR_CUDA;
    } else if (dtype == FLAREPP_F32) {
        rc = simt_cp_partials<float>(s, pl, q, q_shared, k, v, triple, sc.ws, st);
    } else if (dtype == FLAREPP_F16) {
        rc = simt_cp_partials<__half>(s, pl, q, q_shared, k, v, triple, sc.ws, st);
    } else {
        rc = simt_cp_partials<__nv_bfloat16>(s, pl, q, q_shared, k, v, triple, sc.ws, st);
    }
    return sc.release(rc);
}

int cp_merge(const float* gathered, int G, const void* q_fixed, const float* gate, void* state, int B, int H, int M,
             int D, int dtype, void* stream, float* lse_out = nullptr, float* pregate_out = nullptr) {
    const Shape s{B, H, 1, M, D, dtype};
    int rc = check_shape(s);
    if (rc) return rc;
    if (G < 1 || !gathered || !state || (gate && !q_fixed)) return FLAREPP_ERR_INVALID_ARG;
    if (!aligned16(gathered) || !aligned16(state) || (q_fixed && !aligned16(q_fixed)) ||
        (gate && (reinterpret_cast<uintptr_t>(gate) & 3u)))
        return FLAREPP_ERR_INVALID_ARG;
    const int64_t rows = s.bh() * M;
    const size_t gb = (size_t)G * rows * (D + 2) * sizeof(float);
    if (overlaps(state, latent_state_bytes(s), gathered, gb)) return FLAREPP_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    MergeParams mp{};
    mp.part_O = gathered;
    mp.o_part_stride = rows * (D + 2);
    mp.part_ml = reinterpret_cast<const float2*>(gathered + rows * D);
    mp.ml_part_stride = rows * (D + 2) / 2;
    mp.chunks = G;
    mp.B = B; mp.H = H; mp.M = M;
    mp.mode = gate ? kMergeSynthesis : kMergeEncode;
    mp.q_fixed = q_fixed; mp.gate = gate;
    mp.out_f32 = static_cast<float*>(state);
    mp.out_16 = dtype == FLAREPP_F32 ? nullptr : static_cast<char*>(state) + latent_16_offset(s);
    mp.lse_out = lse_out;
    mp.pregate_out = gate ? pregate_out : nullptr;
    if ((lse_out && (overlaps(lse_out, rows * 4, state, latent_state_bytes(s)) ||
                     overlaps(lse_out, rows * 4, gathered, gb))) ||
        (mp.pregate_out && (overlaps(pregate_out, rows * D * 4, state, latent_state_bytes(s)) ||
                            overlaps(pregate_out, rows * D * 4, gathered, gb))))
        return FLAREPP_ERR_INVALID_ARG;
    const dim3 grid((unsigned)((rows + 7) / 8));
#define FLAREPP_CP_MERGE(T)                                                                        \
    switch (D) {                                                                                   \
        case 16: merge_partials<T, 16><<<grid, 256, 0, st>>>(mp); break;                           \
        case 32: merge_partials<T, 32><<<grid, 256, 0, st>>>(mp); break;                           \
        case 64: merge_partials<T, 64><<<grid, 256, 0, st>>>(mp); break;                           \
        default: merge_partials<T, 128><<<grid, 256, 0, st>>>(mp); break;                          \
    }
    if (dtype == FLAREPP_F32) {
        FLAREPP_CP_MERGE(float)
    } else if (dtype == FLAREPP_F16) {
        FLAREPP_CP_MERGE(__half)
    } else {
        FLAREPP_CP_MERGE(__nv_bfloat16)
    }
#undef FLAREPP_CP_MERGE
    return cudaGetLastError() == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
}

int cp_decode(const void* q, int q_shared, const void* z_state, const void* k, void* y, int B, int H, int N, int M,
              int D, int dtype, const flarepp_options_t* opts, void* stream) {
    const Shape s{B, H, N, M, D, dtype};
    Plan pl{};
    int rc = make_plan(s, opts, &pl);
    if (rc) return rc;
    if (!q || !z_state || !k || !y || (q_shared != 0 && q_shared != 1)) return FLAREPP_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(z_state) || !aligned16(k) || !aligned16(y)) return FLAREPP_ERR_INVALID_ARG;
    const size_t tb = s.tok_bytes();
    if (overlaps(y, tb, k, tb) || overlaps(y, tb, z_state, latent_state_bytes(s)) ||
        overlaps(y, tb, q, q_shared ? s.lat_bytes() : latent_state_bytes(s)))
        return FLAREPP_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const char* q16 = q_shared ? static_cast<const char*>(q) : static_cast<const char*>(q) + latent_16_offset(s);
    const char* z16 = static_cast<const char*>(z_state) + latent_16_offset(s);
    if (pl.path == FLAREPP_PATH_TCGEN05) {
        const tc::Problem pr = tc_problem(s, pl);
        rc = dtype == FLAREPP_F16 ? tc::cp_decode<__half>(pr, q16, q_shared, z16, k, y, st)
                                  : tc::cp_decode<__nv_bfloat16>(pr, q16, q_shared, z16, k, y, st);
        return rc ? (rc == 2 ? FLAREPP_ERR_UNSUPPORTED : FLAREPP_ERR_CUDA) : FLAREPP_OK;
    }
    const float* z32 = static_cast<const float*>(z_state);
    if (dtype == FLAREPP_F32) return simt_cp_decode<float>(s, pl, q, q_shared, z32, k, y, st);
    if (dtype == FLAREPP_F16) return simt_cp_decode<__half>(s, pl, q, q_shared, z32, k, y, st);
    return simt_cp_decode<__nv_bfloat16>(s, pl, q, q_shared, z32, k, y, st);
}

// ------------------------------------------------------------------ backward
//
// Gradients of the mixer with respect to all its inputs, for an upstream
// gradient dy of y (the chain rule through each of the three attentions of the
// FLARE.py README's FLARE++ block; kernels in kernels_bwd.cuh).  The forward's
// synthesis and encode passes run again (split + merge, on the forward's own
// kernel family) and keep their per-latent log-sum-exps and the synthesis
// output before the gate; then
//   decode rows     dk_dec, per-token log-sum-exp and <dy, y>
//   decode cols     partials of dq_dec and dz over token chunks     -> reduce: dz, dq, <dz, z>
//   encode cols     dk = dk_dec + dk_enc, dv
//   encode rows     partials of dq_enc                              -> reduce: dq, dq_dyn, <dq_dyn, q_dyn>
//   synthesis cols  dk0 (keys and values terms)
//   synthesis rows  partials of dq0                                 -> reduce: dq0 per batch element
//   batch reduce    dq_fixed, dq0, dgate (sums over the batch)
// With the gate closed (FLARE) the synthesis stages are skipped and the batch
// reduce gives dq_fixed only.
//
// On the tensor-core path (16-bit I/O with the tcgen05 forward) the forward's
// decode runs too, writing per token the log-sum-exp and <dy, y> instead of y,
// and every token-sum and latent-sum step is one launch of bwd_tc::bwd_kernel
// (kernels_bwd_tc.cuh), the token sides of the decode and the encode fused in
// one; the reduces also write 16-bit copies of dz and dq_dyn (tensor-core
// operands) and the padded (log-sum-exp, Delta) pairs of the next pass.
struct BwdPlan {
    Plan fwd;
    bool tc;                     // tensor-core backward
    int chunks, chunk_len, row_blocks;
    int64_t tok_blocks;
    int64_t n_pad, m_pad;        // strides of the padded statistics (multiples of the column tile)
    size_t off_lse_syn, off_lse_enc, off_qdyn, off_lse_tok, off_delta_tok, off_dk_acc, off_part1, off_part2, off_dz,
        off_dq, off_dqdyn, off_delta_enc, off_delta0, off_dq0b, off_stats_tok, off_stats_enc, off_stats_syn,
        off_dz16, off_dqdyn16, total;
};

int make_bwd_plan(const Shape& s, const flarepp_options_t* o, BwdPlan* bp) {
    int rc = make_plan(s, o, &bp->fwd);
    if (rc) return rc;
    const int G = s.D >= 64 ? s.D / 32 : 1;           // bwd::Lanes<D>::G
    const int rows_per_cta = bwd::kThreads / G;
    const int tile = 4096 / s.D;                       // bwd::Lanes<D>::TILE
    bp->row_blocks = (s.M + rows_per_cta - 1) / rows_per_cta;
    bp->tok_blocks = (s.N + (int64_t)rows_per_cta - 1) / rows_per_cta;
    const int64_t tiles = (s.N + tile - 1) / tile;
    bp->tc = bp->fwd.path == FLAREPP_PATH_TCGEN05;
    const int force = o ? o->force_chunks : 0;
    if (bp->tc) {
        // the latent-row passes split the tokens in chunks of a multiple of 64
        bp->chunk_len = bwd_tc::plan_chunk_len(s.B, s.H, s.M, s.N, s.D, force);
        bp->chunks = bwd_tc::chunks_of(s.N, bp->chunk_len);
    } else {
        int64_t chunks;
        if (force > 0) {
            chunks = std::min<int64_t>(force, tiles);
        } else {
            // about eight CTAs per SM over the latent-side grid, chunks of >= 1 tile
            const int64_t target = 8 * kNumSMs, per = s.bh() * bp->row_blocks;
            chunks = std::max<int64_t>(1, std::min<int64_t>((target + per - 1) / per, tiles));
        }
        const int64_t tiles_per_chunk = (tiles + chunks - 1) / chunks;
        bp->chunk_len = (int)std::min<int64_t>(tiles_per_chunk * tile, INT32_MAX);
        bp->chunks = (int)((s.N + (int64_t)bp->chunk_len - 1) / bp->chunk_len);
    }
    // per-token statistics are read in 32-column tiles, per-latent ones in up to 64
    const int64_t kt = bwd_tc::kKT, ktw = bwd_tc::kKTWide;
    bp->n_pad = (s.N + kt - 1) / kt * kt;
    bp->m_pad = (s.M + ktw - 1) / ktw * ktw;
    const size_t lat = (size_t)s.bh() * s.M, latd = lat * s.D, tok = (size_t)s.bh() * s.N;
    const size_t tc_on = bp->tc ? 1 : 0, simt_on = 1 - tc_on;
    size_t off = bp->fwd.total;
    bp->off_lse_syn = off;   off = align_up(off + lat * sizeof(float));
    bp->off_lse_enc = off;   off = align_up(off + lat * sizeof(float));
    bp->off_qdyn = off;      off = align_up(off + latd * sizeof(float));
    bp->off_lse_tok = off;   off = align_up(off + simt_on * tok * sizeof(float));
    bp->off_delta_tok = off; off = align_up(off + simt_on * tok * sizeof(float));
    bp->off_stats_tok = off; off = align_up(off + tc_on * (size_t)s.bh() * bp->n_pad * sizeof(float2));
    bp->off_stats_enc = off; off = align_up(off + tc_on * (size_t)s.bh() * bp->m_pad * sizeof(float2));
    bp->off_stats_syn = off; off = align_up(off + tc_on * (size_t)s.bh() * bp->m_pad * sizeof(float2));
    bp->off_dz16 = off;      off = align_up(off + tc_on * latd * sizeof(uint16_t));
    bp->off_dqdyn16 = off;   off = align_up(off + tc_on * latd * sizeof(uint16_t));
    bp->off_dk_acc = off;    off = align_up(off + simt_on * tok * s.D * sizeof(float));
    bp->off_part1 = off;     off = align_up(off + (size_t)bp->chunks * latd * sizeof(float));
    bp->off_part2 = off;     off = align_up(off + (size_t)bp->chunks * latd * sizeof(float));
    bp->off_dz = off;        off = align_up(off + latd * sizeof(float));
    bp->off_dq = off;        off = align_up(off + latd * sizeof(float));
    bp->off_dqdyn = off;     off = align_up(off + latd * sizeof(float));
    bp->off_delta_enc = off; off = align_up(off + lat * sizeof(float));
    bp->off_delta0 = off;    off = align_up(off + lat * sizeof(float));
    bp->off_dq0b = off;      off = align_up(off + latd * sizeof(float));
    bp->total = off;
    return FLAREPP_OK;
}

struct BwdArgs {
    const void *q0, *q_fixed, *k0, *k, *v, *dy;
    const float* gate;
    float *dq0, *dq_fixed, *dgate;
    void *dk0, *dk, *dv;
};

int check_bwd_pointers(const Shape& s, const BwdArgs& a) {
    const bool gated = a.gate != nullptr;
    if (!a.q_fixed || !a.k || !a.v || !a.dy || !a.dq_fixed || !a.dk || !a.dv) return FLAREPP_ERR_INVALID_ARG;
    if (gated && (!a.q0 || !a.k0 || !a.dq0 || !a.dgate || !a.dk0)) return FLAREPP_ERR_INVALID_ARG;
    const void* tensors[] = {a.q_fixed, a.k, a.v, a.dy, a.dq_fixed, a.dk, a.dv, gated ? a.q0 : nullptr,
                             gated ? a.k0 : nullptr, gated ? a.dq0 : nullptr, gated ? a.dk0 : nullptr};
    for (const void* t : tensors)
        if (t && !aligned16(t)) return FLAREPP_ERR_INVALID_ARG;
    if (gated && ((reinterpret_cast<uintptr_t>(a.gate) & 3u) || (reinterpret_cast<uintptr_t>(a.dgate) & 3u)))
        return FLAREPP_ERR_INVALID_ARG;
    const size_t tb = s.tok_bytes(), lb = s.lat_bytes(), l32 = (size_t)s.H * s.M * s.D * sizeof(float);
    const size_t gb = (size_t)s.H * sizeof(float);
    struct Span { const void* p; size_t n; };
    const Span ins[] = {{a.q_fixed, lb}, {a.k, tb}, {a.v, tb}, {a.dy, tb}, {gated ? a.q0 : nullptr, lb},
                        {gated ? a.k0 : nullptr, tb}, {gated ? a.gate : nullptr, gb}};
    const Span outs[] = {{a.dq_fixed, l32}, {a.dk, tb}, {a.dv, tb}, {gated ? a.dq0 : nullptr, l32},
                         {gated ? a.dgate : nullptr, gb}, {gated ? a.dk0 : nullptr, tb}};
    for (const Span& o : outs) {
        for (const Span& i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return FLAREPP_ERR_INVALID_ARG;
        for (const Span& o2 : outs)
            if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return FLAREPP_ERR_INVALID_ARG;
    }
    return FLAREPP_OK;
}

// Launches with programmatic stream serialization (every backward kernel calls
// pdl_wait() before its first global access); keeps the first launch error.
struct BwdLauncher {
    cudaStream_t st;
    cudaError_t err = cudaSuccess;
    template <typename K, typename... Args>
    void operator()(K kern, dim3 grid, dim3 block, Args... args) {
        const cudaError_t e = tc::launch_pdl(kern, grid, block, 0, st, args...);
        if (err == cudaSuccess) err = e;
    }
};

// The backward launches for one I/O type T, one latent-operand type TQ of the
// decode and encode (T, or fp32 when the forward's SIMT kernels ran the
// encode from fp32 routing queries) and one head dim D.
template <typename T, typename TQ, int D>
cudaError_t run_backward(const Shape& s, const BwdPlan& bp, const BwdArgs& a, char* ws, const void* q_lat, int q_bh,
                         StageEvents& ev, cudaStream_t st) {
    const bool gated = a.gate != nullptr;
    BwdLauncher launch_bwd_kernel{st};
    const Plan& pl = bp.fwd;
    bwd::Params p{};
    p.B = s.B; p.H = s.H; p.N = s.N; p.M = s.M;
    p.tok_row = pl.tok.row; p.tok_h = pl.tok.h; p.tok_b = pl.tok.b;
    p.scale_log2 = pl.scale_log2;
    p.scale = pl.scale_log2 / kLog2e;
    p.chunks = bp.chunks; p.chunk_len = bp.chunk_len;
    p.lse_tok = reinterpret_cast<float*>(ws + bp.off_lse_tok);
    p.delta_tok = reinterpret_cast<float*>(ws + bp.off_delta_tok);
    p.dk_acc = reinterpret_cast<float*>(ws + bp.off_dk_acc);
    p.part1 = reinterpret_cast<float*>(ws + bp.off_part1);
    p.part2 = reinterpret_cast<float*>(ws + bp.off_part2);
    float* z32 = reinterpret_cast<float*>(ws + pl.off_z32);
    float* dz = reinterpret_cast<float*>(ws + bp.off_dz);
    float* dq = reinterpret_cast<float*>(ws + bp.off_dq);
    float* dqdyn = reinterpret_cast<float*>(ws + bp.off_dqdyn);
    float* qdyn = reinterpret_cast<float*>(ws + bp.off_qdyn);
    float* delta_enc = reinterpret_cast<float*>(ws + bp.off_delta_enc);
    float* delta0 = reinterpret_cast<float*>(ws + bp.off_delta0);
    float* dq0b = reinterpret_cast<float*>(ws + bp.off_dq0b);
    const dim3 tok_grid((unsigned)bp.tok_blocks, (unsigned)s.bh());
    const dim3 lat_grid((unsigned)bp.chunks, (unsigned)s.bh(), (unsigned)bp.row_blocks);
    const int64_t rows = s.bh() * s.M;
    const dim3 red_grid((unsigned)((rows + 7) / 8));

    // decode: y = SDPA(k, q, z)
    p.Qlat = q_lat; p.q_batch_heads = q_bh; p.Zlat = z32;
    p.Ktok = a.k; p.Vtok = nullptr; p.dYtok = a.dy;
    launch_bwd_kernel(bwd::decode_rows<T, TQ, D>, tok_grid, dim3(bwd::kThreads), p);
    ev.mark(st);
    launch_bwd_kernel(bwd::decode_cols<T, TQ, D>, lat_grid, dim3(bwd::kThreads), p);
    ev.mark(st);
    bwd::ReduceParams rp{};
    rp.part1 = p.part1; rp.part2 = p.part2; rp.chunks = bp.chunks;
    rp.B = s.B; rp.H = s.H; rp.M = s.M; rp.scale = p.scale;
    rp.mode = bwd::kReduceDecode; rp.z = z32; rp.dz = dz; rp.dq = dq; rp.delta = delta_enc;
    launch_bwd_kernel(bwd::reduce_partials<float, D>, red_grid, dim3(256), rp);
    ev.mark(st);

    // encode: z = SDPA(q, k, v)
    p.dOlat = dz; p.lse_lat = reinterpret_cast<float*>(ws + bp.off_lse_enc); p.delta_lat = delta_enc;
    p.Ktok = a.k; p.Vtok = a.v; p.dK = a.dk; p.dV = a.dv;
    launch_bwd_kernel(bwd::token_cols<T, TQ, D>, tok_grid, dim3(bwd::kThreads), p);
    ev.mark(st);
    launch_bwd_kernel(bwd::latent_rows<T, TQ, D>, lat_grid, dim3(bwd::kThreads), p);
    ev.mark(st);
    rp.mode = bwd::kReduceEncode; rp.gate = a.gate; rp.qdyn = qdyn; rp.dqdyn = dqdyn; rp.delta = delta0;
    launch_bwd_kernel(bwd::reduce_partials<float, D>, red_grid, dim3(256), rp);
    ev.mark(st);

    if (gated) {
        // synthesis: q_dyn = SDPA(q0, k0, k0), output gradient dq_dyn = gate * dq
        p.Qlat = a.q0; p.q_batch_heads = 0;
        p.dOlat = dqdyn; p.lse_lat = reinterpret_cast<float*>(ws + bp.off_lse_syn); p.delta_lat = delta0;
        p.Ktok = a.k0; p.Vtok = a.k0; p.dK = a.dk0; p.dV = nullptr;
        launch_bwd_kernel(bwd::token_cols<T, T, D>, tok_grid, dim3(bwd::kThreads), p);
        ev.mark(st);
        launch_bwd_kernel(bwd::latent_rows<T, T, D>, lat_grid, dim3(bwd::kThreads), p);
        ev.mark(st);
        rp.mode = bwd::kReduceSynthesis; rp.dq0b = dq0b;
        launch_bwd_kernel(bwd::reduce_partials<float, D>, red_grid, dim3(256), rp);
        ev.mark(st);
    }
    bwd::BatchParams bt{};
    bt.B = s.B; bt.H = s.H; bt.M = s.M;
    bt.dq = dq; bt.dq_fixed = a.dq_fixed;
    if (gated) { bt.dq0b = dq0b; bt.qdyn = qdyn; bt.dq0 = a.dq0; bt.dgate = a.dgate; }
    launch_bwd_kernel(bwd::reduce_batch<D>, dim3((unsigned)s.H), dim3(256), bt);
    ev.mark(st);
    return launch_bwd_kernel.err;
}

// The tensor-core backward after the recomputed forward (which has left q, z,
// their 16-bit copies, the log-sum-exps, q_dyn and the per-token statistics
// in the workspace).
template <typename E, int D>
cudaError_t run_backward_tc(const Shape& s, const BwdPlan& bp, const BwdArgs& a, char* ws, StageEvents& ev,
                            cudaStream_t st) {
    using bwd_tc::Operand;
    const bool gated = a.gate != nullptr;
    const Plan& pl = bp.fwd;
    const float scale = pl.scale_log2 / kLog2e;
    cudaError_t err = cudaSuccess;
    auto note = [&](int rc) {
        if (rc && err == cudaSuccess) err = cudaErrorLaunchFailure;
        ev.mark(st);
    };
    float2* stats_tok = reinterpret_cast<float2*>(ws + bp.off_stats_tok);
    float2* stats_enc = reinterpret_cast<float2*>(ws + bp.off_stats_enc);
    float2* stats_syn = reinterpret_cast<float2*>(ws + bp.off_stats_syn);
    float* part1 = reinterpret_cast<float*>(ws + bp.off_part1);
    float* part2 = reinterpret_cast<float*>(ws + bp.off_part2);
    const Operand q_lat = gated ? Operand{ws + pl.off_q16, false, false} : Operand{a.q_fixed, false, true};
    const Operand z_lat{ws + pl.off_z16, false, false};
    const Operand dz_lat{ws + bp.off_dz16, false, false};
    const Operand dqdyn_lat{ws + bp.off_dqdyn16, false, false};
    const Operand q0{a.q0, false, true};
    const Operand k{a.k, true, false}, v{a.v, true, false}, dy{a.dy, true, false}, k0{a.k0, true, false};

    bwd_tc::Launch base{};
    base.B = s.B; base.H = s.H; base.N = s.N; base.M = s.M; base.D = s.D;
    base.tok = pl.tok;
    base.scale_log2 = pl.scale_log2;
    base.scale = scale;
    base.chunk_len = bp.chunk_len;
    auto latent_rows = [&](Operand A, Operand C, Operand Bc, Operand Ec, bool acc2, bool col_stats,
                           const float2* stats, int64_t stride) {
        bwd_tc::Launch L = base;
        L.a = A; L.c = C; L.b = Bc; L.e = Ec;
        L.rows_tok = false; L.has_acc2 = acc2; L.stats_per_col = col_stats;
        L.stats = stats; L.stats_stride = stride;
        L.epi = bwd_tc::kEpiPartials; L.part1 = part1; L.part2 = part2;
        note(bwd_tc::launch_bwd_d<E>(L, st));
    };
    auto token_rows = [&](Operand A, Operand C, Operand Bc, Operand Ec, bool acc2, bool col_stats,
                          const float2* stats, int64_t stride, int epi, void* out1, void* out2) {
        bwd_tc::Launch L = base;
        L.a = A; L.c = C; L.b = Bc; L.e = Ec;
        L.rows_tok = true; L.has_acc2 = acc2; L.stats_per_col = col_stats;
        L.stats = stats; L.stats_stride = stride;
        L.epi = epi; L.out1 = out1; L.out2 = out2;
        note(bwd_tc::launch_bwd_d<E>(L, st));
    };
    BwdLauncher launch{st};
    const int64_t rows = s.bh() * s.M;
    const dim3 red_grid((unsigned)((rows + 7) / 8));
    bwd::ReduceParams rp{};
    rp.part1 = part1; rp.part2 = part2; rp.chunks = bp.chunks;
    rp.B = s.B; rp.H = s.H; rp.M = s.M; rp.scale = scale;
    rp.stats_stride = bp.m_pad;
    float* z32 = reinterpret_cast<float*>(ws + pl.off_z32);
    float* dq = reinterpret_cast<float*>(ws + bp.off_dq);
    float* qdyn = reinterpret_cast<float*>(ws + bp.off_qdyn);
    float* dq0b = reinterpret_cast<float*>(ws + bp.off_dq0b);

    // decode y = SDPA(k, q, z): latent side (dq_dec, dz partials)
    latent_rows(q_lat, z_lat, k, dy, true, true, stats_tok, bp.n_pad);
    rp.mode = bwd::kReduceDecode; rp.z = z32; rp.dz = reinterpret_cast<float*>(ws + bp.off_dz); rp.dq = dq;
    rp.delta = reinterpret_cast<float*>(ws + bp.off_delta_enc);
    rp.out16 = ws + bp.off_dz16; rp.stats_out = stats_enc; rp.lse_in = reinterpret_cast<float*>(ws + bp.off_lse_enc);
    launch(bwd::reduce_partials<E, D>, red_grid, dim3(256), rp);
    ev.mark(st);
    // the token sides of the decode and the encode in one launch (they share S = k q^T
    // and the product with q): dk = dk_dec + dk_enc and dv
    {
        bwd_tc::Launch L = base;
        L.a = k; L.c = dy; L.c2 = v; L.b = q_lat; L.e = z_lat; L.e2 = dz_lat;
        L.dual = true; L.rows_tok = true; L.has_acc2 = true; L.stats_per_col = false;
        L.stats = stats_tok; L.stats_stride = bp.n_pad;      // the decode's softmax: per token
        L.stats2 = stats_enc; L.stats2_stride = bp.m_pad;    // the encode's: per latent
        L.epi = bwd_tc::kEpiTokDkDv; L.out1 = a.dk; L.out2 = a.dv;
        note(bwd_tc::launch_bwd_d<E>(L, st));
    }
    // encode z = SDPA(q, k, v): latent side (dq_enc partials)
    latent_rows(q_lat, dz_lat, k, v, false, false, stats_enc, bp.m_pad);
    rp.mode = bwd::kReduceEncode; rp.gate = a.gate; rp.qdyn = qdyn;
    rp.dqdyn = reinterpret_cast<float*>(ws + bp.off_dqdyn); rp.delta = reinterpret_cast<float*>(ws + bp.off_delta0);
    rp.out16 = ws + bp.off_dqdyn16; rp.stats_out = gated ? stats_syn : nullptr;
    rp.lse_in = reinterpret_cast<float*>(ws + bp.off_lse_syn);
    launch(bwd::reduce_partials<E, D>, red_grid, dim3(256), rp);
    ev.mark(st);
    if (gated) {
        // synthesis q_dyn = SDPA(q0, k0, k0) with output gradient dq_dyn = gate dq
        token_rows(k0, k0, q0, dqdyn_lat, true, true, stats_syn, bp.m_pad, bwd_tc::kEpiTokDk0, a.dk0, nullptr);
        latent_rows(q0, dqdyn_lat, k0, k0, false, false, stats_syn, bp.m_pad);
        rp.mode = bwd::kReduceSynthesis; rp.dq0b = dq0b; rp.out16 = nullptr; rp.stats_out = nullptr;
        launch(bwd::reduce_partials<E, D>, red_grid, dim3(256), rp);
        ev.mark(st);
    }
    bwd::BatchParams bt{};
    bt.B = s.B; bt.H = s.H; bt.M = s.M;
    bt.dq = dq; bt.dq_fixed = a.dq_fixed;
    if (gated) { bt.dq0b = dq0b; bt.qdyn = qdyn; bt.dq0 = a.dq0; bt.dgate = a.dgate; }
    launch(bwd::reduce_batch<D>, dim3((unsigned)s.H), dim3(256), bt);
    ev.mark(st);
    return err != cudaSuccess ? err : launch.err;
}

template <typename E>
cudaError_t run_backward_tc_d(const Shape& s, const BwdPlan& bp, const BwdArgs& a, char* ws, StageEvents& ev,
                              cudaStream_t st) {
    switch (s.D) {
        case 16: return run_backward_tc<E, 16>(s, bp, a, ws, ev, st);
        case 32: return run_backward_tc<E, 32>(s, bp, a, ws, ev, st);
        case 64: return run_backward_tc<E, 64>(s, bp, a, ws, ev, st);
        default: return run_backward_tc<E, 128>(s, bp, a, ws, ev, st);
    }
}

template <typename T, typename TQ>
cudaError_t run_backward_d(const Shape& s, const BwdPlan& bp, const BwdArgs& a, char* ws, const void* q_lat,
                           int q_bh, StageEvents& ev, cudaStream_t st) {
    switch (s.D) {
        case 16: return run_backward<T, TQ, 16>(s, bp, a, ws, q_lat, q_bh, ev, st);
        case 32: return run_backward<T, TQ, 32>(s, bp, a, ws, q_lat, q_bh, ev, st);
        case 64: return run_backward<T, TQ, 64>(s, bp, a, ws, q_lat, q_bh, ev, st);
        default: return run_backward<T, TQ, 128>(s, bp, a, ws, q_lat, q_bh, ev, st);
    }
}

// ------------------------------------------------------------------ saved forward state
//
// A training step runs the forward and then the backward.  The training forward
// keeps, in a caller-owned context, what the backward would otherwise recompute:
// the routing queries q and the latents z (fp32), the synthesis output before the
// gate, the per-latent log-sum-exps of the synthesis and the encode, and (tensor-
// core path) the decode's per-token log-sum-exp.  The backward given the context
// skips the recomputed forward passes: it rebuilds the 16-bit operand copies of q
// and z by rounding, and takes <dy, y> per token from the forward's output y.
struct Context {
    size_t q32, z32, qdyn, lse_syn, lse_enc, tok, total;
};

Context context_layout(const Shape& s) {
    const size_t lat = (size_t)s.bh() * s.M, latd = lat * s.D;
    const int64_t kt = bwd_tc::kKT, n_pad = (s.N + kt - 1) / kt * kt;
    Context c{};
    size_t off = 0;
    c.q32 = off;     off = align_up(off + latd * sizeof(float));
    c.z32 = off;     off = align_up(off + latd * sizeof(float));
    c.qdyn = off;    off = align_up(off + latd * sizeof(float));
    c.lse_syn = off; off = align_up(off + lat * sizeof(float));
    c.lse_enc = off; off = align_up(off + lat * sizeof(float));
    c.tok = off;     off = align_up(off + (size_t)s.bh() * n_pad * sizeof(float2));
    c.total = off;
    return c;
}

int check_context(const Shape& s, const void* ctx, size_t ctx_bytes) {
    if (!ctx) return FLAREPP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ctx) % kAlign) return FLAREPP_ERR_INVALID_ARG;
    if (ctx_bytes < context_layout(s).total) return FLAREPP_ERR_WORKSPACE;
    return FLAREPP_OK;
}

int forward_train(const void* q0, const void* q_fixed, const float* gate, const void* k0, const void* k,
                  const void* v, void* y, int B, int H, int N, int M, int D, int dtype,
                  const flarepp_options_t* opts, void* ctx, size_t ctx_bytes, void* stream) {
    const Shape s{B, H, N, M, D, dtype};
    int rc = check_shape(s);
    if (rc) return rc;
    rc = check_context(s, ctx, ctx_bytes);
    if (rc) return rc;
    const Context c = context_layout(s);
    char* base = static_cast<char*>(ctx);
    const size_t tb = s.tok_bytes();
    if (overlaps(ctx, c.total, y, tb) || overlaps(ctx, c.total, k, tb) || overlaps(ctx, c.total, v, tb) ||
        overlaps(ctx, c.total, q_fixed, s.lat_bytes()) || (gate && overlaps(ctx, c.total, k0, tb)))
        return FLAREPP_ERR_INVALID_ARG;
    flarepp_options_t o = opts ? *opts : flarepp_options_t{};
    o.q_out = reinterpret_cast<float*>(base + c.q32);
    o.z_out = reinterpret_cast<float*>(base + c.z32);
    Plan pl{};
    rc = make_plan(s, &o, &pl);
    if (rc) return rc;
    FwdExtras ex;
    ex.lse_syn = reinterpret_cast<float*>(base + c.lse_syn);
    ex.lse_enc = reinterpret_cast<float*>(base + c.lse_enc);
    ex.qdyn = reinterpret_cast<float*>(base + c.qdyn);
    if (pl.path == FLAREPP_PATH_TCGEN05) {
        const int64_t kt = bwd_tc::kKT;
        ex.tok_stats = reinterpret_cast<float2*>(base + c.tok);
        ex.tok_stats_stride = (s.N + kt - 1) / kt * kt;
    }
    return forward(q0, q_fixed, gate, k0, k, v, y, B, H, N, M, D, dtype, &o, stream, ex);
}

// Fills the backward's workspace regions from a saved context: the plain copies
// (cudaMemcpyAsync), the 16-bit operand copies of q and z (tensor-core path),
// and <dy, y> per token.
template <typename E, int D>
int restore_context(const Shape& s, const BwdPlan& bp, const BwdArgs& a, const void* y, const char* ctx, char* ws,
                    StageEvents& ev, cudaStream_t st) {
    const Plan& pl = bp.fwd;
    const Context c = context_layout(s);
    const size_t lat = (size_t)s.bh() * s.M, latd = lat * s.D;
    ev.mark(st);        // before the first launch, as the recomputed forward does
    bool ok = cudaMemcpyAsync(ws + pl.off_q32, ctx + c.q32, latd * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess &&
              cudaMemcpyAsync(ws + pl.off_z32, ctx + c.z32, latd * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess &&
              cudaMemcpyAsync(ws + bp.off_lse_enc, ctx + c.lse_enc, lat * 4, cudaMemcpyDeviceToDevice, st) ==
                  cudaSuccess;
    if (ok && a.gate)
        ok = cudaMemcpyAsync(ws + bp.off_qdyn, ctx + c.qdyn, latd * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess &&
             cudaMemcpyAsync(ws + bp.off_lse_syn, ctx + c.lse_syn, lat * 4, cudaMemcpyDeviceToDevice, st) ==
                 cudaSuccess;
    if (!ok) return FLAREPP_ERR_CUDA;
    if (bp.tc) {
        ok = cudaMemcpyAsync(ws + bp.off_stats_tok, ctx + c.tok, (size_t)s.bh() * bp.n_pad * sizeof(float2),
                             cudaMemcpyDeviceToDevice, st) == cudaSuccess;
        if (!ok) return FLAREPP_ERR_CUDA;
        const unsigned rgrid = (unsigned)std::min<int64_t>((int64_t)((latd / 8 + 255) / 256), (int64_t)kNumSMs * 8);
        bwd::round_to_io<E><<<rgrid, 256, 0, st>>>(reinterpret_cast<const float*>(ctx + c.q32),
                                                   reinterpret_cast<E*>(ws + pl.off_q16), (int64_t)latd);
        bwd::round_to_io<E><<<rgrid, 256, 0, st>>>(reinterpret_cast<const float*>(ctx + c.z32),
                                                   reinterpret_cast<E*>(ws + pl.off_z16), (int64_t)latd);
        ev.mark(st);
        const int64_t rows = s.bh() * s.N;
        const int rw = 32 / (D * 2 / 16);
        const int64_t want = (rows + 8 * rw - 1) / (8 * rw);
        bwd::token_delta<E, D><<<(unsigned)std::min<int64_t>(want, (int64_t)kNumSMs * 16), 256, 0, st>>>(
            reinterpret_cast<float2*>(ws + bp.off_stats_tok), bp.n_pad, static_cast<const E*>(a.dy),
            static_cast<const E*>(y), s.H, s.N, rows, pl.tok.row, pl.tok.h, pl.tok.b);
        ev.mark(st);
    }
    return cudaGetLastError() == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
}

template <typename E>
int restore_context_d(const Shape& s, const BwdPlan& bp, const BwdArgs& a, const void* y, const char* ctx, char* ws,
                      StageEvents& ev, cudaStream_t st) {
    switch (s.D) {
        case 16: return restore_context<E, 16>(s, bp, a, y, ctx, ws, ev, st);
        case 32: return restore_context<E, 32>(s, bp, a, y, ctx, ws, ev, st);
        case 64: return restore_context<E, 64>(s, bp, a, y, ctx, ws, ev, st);
        default: return restore_context<E, 128>(s, bp, a, y, ctx, ws, ev, st);
    }
}

// Gradient through the synthesis normalisation (norm_synthesis): dk0 (I/O
// dtype, token rows) and dq0 (fp32 [H,M,D]) were taken with respect to the
// normalised rows; map them to the raw q0, k0 rows in place.
template <typename T, int D>
void launch_rms_backward(const Shape& s, const BwdArgs& a, StageEvents& ev, cudaStream_t st) {
    const int64_t rows_k = s.bh() * s.N, rows_q = (int64_t)s.H * s.M;
    const int rw = 32 / (D * (int)sizeof(T) / 16);                  // rows per warp pass
    const int64_t want = (rows_k + 8 * rw - 1) / (8 * rw);
    bwd::rms_backward_rows_coop<T, D><<<(unsigned)std::min<int64_t>(want, (int64_t)kNumSMs * 16), 256, 0, st>>>(
        static_cast<const T*>(a.k0), static_cast<T*>(a.dk0), rows_k, kNormEps);
    ev.mark(st);
    bwd::rms_backward_rows<T, float, D><<<(unsigned)((rows_q + 255) / 256), 256, 0, st>>>(
        static_cast<const T*>(a.q0), a.dq0, rows_q, kNormEps);
    ev.mark(st);
}

template <typename T>
void rms_backward(const Shape& s, const BwdArgs& a, StageEvents& ev, cudaStream_t st) {
    switch (s.D) {
        case 16: launch_rms_backward<T, 16>(s, a, ev, st); break;
        case 32: launch_rms_backward<T, 32>(s, a, ev, st); break;
        case 64: launch_rms_backward<T, 64>(s, a, ev, st); break;
        default: launch_rms_backward<T, 128>(s, a, ev, st); break;
    }
}

int backward(const BwdArgs& a, int B, int H, int N, int M, int D, int dtype, const flarepp_options_t* opts,
             void* stream, const void* ctx = nullptr, size_t ctx_bytes = 0, const void* y = nullptr) {
    const Shape s{B, H, N, M, D, dtype};
    BwdPlan bp{};
    int rc = make_bwd_plan(s, opts, &bp);
    if (rc) return rc;
    rc = check_bwd_pointers(s, a);
    if (rc) return rc;
    const Plan& pl = bp.fwd;
    const bool gated = a.gate != nullptr;
    if (ctx) {
        rc = check_context(s, ctx, ctx_bytes);
        if (rc) return rc;
        if (!y || !aligned16(y)) return FLAREPP_ERR_INVALID_ARG;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* ws = nullptr;
    bool owned = false;
    if (opts && opts->workspace) {
        if (opts->workspace_bytes < bp.total) return FLAREPP_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(opts->workspace) % kAlign) return FLAREPP_ERR_INVALID_ARG;
        ws = static_cast<char*>(opts->workspace);
    } else {
        if (cudaMallocAsync(reinterpret_cast<void**>(&ws), bp.total, st) != cudaSuccess) {
            cudaGetLastError();
            return FLAREPP_ERR_WORKSPACE;
        }
        owned = true;
    }
    StageEvents ev;
    if (opts && opts->n_stage_events > 0) {
        ev.ev = opts->stage_events;
        ev.n = opts->n_stage_events;
    }
    // the forward's synthesis and encode, keeping what the backward needs
    FwdExtras ex;
    ex.lse_syn = reinterpret_cast<float*>(ws + bp.off_lse_syn);
    ex.lse_enc = reinterpret_cast<float*>(ws + bp.off_lse_enc);
    ex.qdyn = reinterpret_cast<float*>(ws + bp.off_qdyn);
    ex.decode = bp.tc;      // the tensor-core path takes the per-token statistics from the forward's decode
    if (bp.tc) {
        ex.tok_stats = reinterpret_cast<float2*>(ws + bp.off_stats_tok);
        ex.tok_stats_stride = bp.n_pad;
        ex.dy = a.dy;
    }
    // with norm_synthesis the synthesis (forward and backward) reads normalised
    // copies of q0 and k0, and dq0, dk0 are mapped back through the step at the end
    const bool norm = pl.norm_synthesis && gated;
    BwdArgs an = a;
    if (norm) {
        ev.mark(st);
        rms_norm(s, a.q0, ws + pl.off_q0n, a.k0, ws + pl.off_k0n, st);
        an.q0 = ws + pl.off_q0n;
        an.k0 = ws + pl.off_k0n;
    }
    if (ctx) {
        // the training forward's saved state replaces the recomputed passes
        const char* c = static_cast<const char*>(ctx);
        if (dtype == FLAREPP_F16) rc = restore_context_d<__half>(s, bp, an, y, c, ws, ev, st);
        else if (dtype == FLAREPP_BF16) rc = restore_context_d<__nv_bfloat16>(s, bp, an, y, c, ws, ev, st);
        else rc = restore_context_d<float>(s, bp, an, y, c, ws, ev, st);
    } else {
        rc = run(s, pl, an.q0, an.q_fixed, an.gate, an.k0, an.k, an.v, nullptr, ws, nullptr, nullptr, ev, st, ex);
    }
    if (rc == FLAREPP_OK && bp.tc) {
        cudaError_t e;
        if (dtype == FLAREPP_F16) e = run_backward_tc_d<__half>(s, bp, an, ws, ev, st);
        else e = run_backward_tc_d<__nv_bfloat16>(s, bp, an, ws, ev, st);
        rc = (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? FLAREPP_OK : FLAREPP_ERR_CUDA;
    } else if (rc == FLAREPP_OK) {
        // the routing queries the forward's encode read: q_fixed with the gate
        // closed; else the I/O-dtype copy (tensor cores) or fp32 (SIMT)
        const bool q_f32 = gated && (pl.path == FLAREPP_PATH_SIMT || dtype == FLAREPP_F32);
        const void* q_lat = !gated ? a.q_fixed : q_f32 ? static_cast<const void*>(ws + pl.off_q32)
                                                       : static_cast<const void*>(ws + pl.off_q16);
        const int q_bh = gated ? s.H : 0;
        cudaError_t e;
        if (dtype == FLAREPP_F32) e = run_backward_d<float, float>(s, bp, an, ws, q_lat, q_bh, ev, st);
        else if (dtype == FLAREPP_F16 && q_f32) e = run_backward_d<__half, float>(s, bp, an, ws, q_lat, q_bh, ev, st);
        else if (dtype == FLAREPP_F16) e = run_backward_d<__half, __half>(s, bp, an, ws, q_lat, q_bh, ev, st);
        else if (q_f32) e = run_backward_d<__nv_bfloat16, float>(s, bp, an, ws, q_lat, q_bh, ev, st);
        else e = run_backward_d<__nv_bfloat16, __nv_bfloat16>(s, bp, an, ws, q_lat, q_bh, ev, st);
        if (cudaGetLastError() != cudaSuccess) e = cudaErrorLaunchFailure;
        rc = e == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
    }
    if (rc == FLAREPP_OK && norm) {
        if (dtype == FLAREPP_F32) rms_backward<float>(s, a, ev, st);
        else if (dtype == FLAREPP_F16) rms_backward<__half>(s, a, ev, st);
        else rms_backward<__nv_bfloat16>(s, a, ev, st);
        rc = cudaGetLastError() == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
    }
    if (owned && cudaFreeAsync(ws, st) != cudaSuccess && rc == FLAREPP_OK) rc = FLAREPP_ERR_CUDA;
    return rc;
}

// ------------------------------------------------------------------ token-sharded backward
//
// The backward with the N tokens split across ranks (physicsnemo issue #2024,
// section 2: the distributed encoder and its backward).  Every sum over
// tokens in the backward is a sum of per-rank partial sums; every sum over
// latents stays local.  So each rank runs the single-GPU steps on its tokens,
// and where the single-GPU backward reduces token-chunk partials, a rank
// reduces its own chunks into a latent-sized fp32 region of its state that the
// caller sums over the ranks (an all-reduce) before the next stage:
//   stage 1  decode: per-token statistics, latent side        -> region 1 = (dq_dec, dz)
//   stage 2  dz, <dz, z>; token sides of decode + encode (dk, dv); latent side of the encode
//                                                             -> region 2 = dq_enc
//   stage 3  dq = dq_dec + dq_enc, dq_dyn = gate dq; token side of the synthesis (dk0);
//            latent side of the synthesis                     -> region 3 = dq0 per batch element
//   stage 4  batch reduce: dq_fixed, dq0, dgate (identical on every rank)
// The forward's merged latent states (flarepp_cp_merge) provide q and z, and
// flarepp_cp_merge_ex the per-latent log-sum-exps and the pre-gate q_dyn.
struct CpLayout {
    size_t r1, r2, r3, ws, total;
};

CpLayout cp_layout(const Shape& s, const BwdPlan& bp) {
    const size_t latd = (size_t)s.bh() * s.M * s.D * sizeof(float);
    CpLayout L{};
    size_t off = 0;
    L.r1 = off; off = align_up(off + 2 * latd);        // dq_dec, dz
    L.r2 = off; off = align_up(off + latd);            // dq_enc
    L.r3 = off; off = align_up(off + latd);            // dq0 per batch element
    L.ws = off; off = align_up(off + bp.total);        // the backward's workspace
    L.total = off;
    return L;
}

struct CpBwdArgs {
    BwdArgs a;
    const void* q_state;     // gated: the routing-query state (fp32 rows, then the I/O-dtype copy)
    const void* z_state;     // the latent state
    const float *lse_syn, *lse_enc, *qdyn;
};

template <typename T, int D>
cudaError_t cp_stage(int stage, const Shape& s, const BwdPlan& bp, const CpBwdArgs& c, char* state,
                     StageEvents& ev, cudaStream_t st) {
    const BwdArgs& a = c.a;
    const bool gated = a.gate != nullptr;
    const Plan& pl = bp.fwd;
    const bool tcp = bp.tc;
    const CpLayout L = cp_layout(s, bp);
    char* ws = state + L.ws;
    const int64_t latd = s.bh() * s.M * s.D;
    float* r1q = reinterpret_cast<float*>(state + L.r1);
    float* r1z = r1q + latd;
    float* r2 = reinterpret_cast<float*>(state + L.r2);
    float* r3 = reinterpret_cast<float*>(state + L.r3);
    const float scale = pl.scale_log2 / kLog2e;
    const size_t o16 = latent_16_offset(s);
    const float* z32 = static_cast<const float*>(c.z_state);
    const char* z16 = static_cast<const char*>(c.z_state) + o16;
    float* dz = reinterpret_cast<float*>(ws + bp.off_dz);
    float* dq = reinterpret_cast<float*>(ws + bp.off_dq);
    float* dqdyn = reinterpret_cast<float*>(ws + bp.off_dqdyn);
    float* delta_enc = reinterpret_cast<float*>(ws + bp.off_delta_enc);
    float* delta0 = reinterpret_cast<float*>(ws + bp.off_delta0);
    float* dq0b = reinterpret_cast<float*>(ws + bp.off_dq0b);
    float* part1 = reinterpret_cast<float*>(ws + bp.off_part1);
    float* part2 = reinterpret_cast<float*>(ws + bp.off_part2);
    float2* stats_tok = reinterpret_cast<float2*>(ws + bp.off_stats_tok);
    float2* stats_enc = reinterpret_cast<float2*>(ws + bp.off_stats_enc);
    float2* stats_syn = reinterpret_cast<float2*>(ws + bp.off_stats_syn);
    // the synthesis reads normalised copies of q0, k0 with norm_synthesis
    const bool norm = pl.norm_synthesis && gated;
    const void* q0s = norm ? static_cast<const void*>(ws + pl.off_q0n) : a.q0;
    const void* k0s = norm ? static_cast<const void*>(ws + pl.off_k0n) : a.k0;

    BwdLauncher launch{st};
    const dim3 red_grid((unsigned)((s.bh() * s.M + 7) / 8));
    bwd::ReduceParams rp{};
    rp.B = s.B; rp.H = s.H; rp.M = s.M;
    auto reduce = [&](const bwd::ReduceParams& r) {
        launch(bwd::reduce_partials<T, D>, red_grid, dim3(256), r);
        ev.mark(st);
    };
    cudaError_t err = cudaSuccess;
    auto note = [&](int rc) {
        if (rc && err == cudaSuccess) err = cudaErrorLaunchFailure;
        ev.mark(st);
    };

    // ---- the kernel families' steps (the tensor-core path for 16-bit I/O with the
    // tcgen05 forward, else SIMT), with the same operands as the single-GPU backward
    using bwd_tc::Operand;
    bwd_tc::Launch base{};
    base.B = s.B; base.H = s.H; base.N = s.N; base.M = s.M; base.D = s.D;
    base.tok = pl.tok; base.scale_log2 = pl.scale_log2; base.scale = scale; base.chunk_len = bp.chunk_len;
    const Operand q_lat = gated ? Operand{static_cast<const char*>(c.q_state) + o16, false, false}
                                : Operand{a.q_fixed, false, true};
    const Operand z_lat{z16, false, false};
    const Operand k{a.k, true, false}, v{a.v, true, false}, dyo{a.dy, true, false}, k0o{k0s, true, false};
    const Operand q0o{q0s, false, true};
    const Operand dz_lat{ws + bp.off_dz16, false, false}, dqdyn_lat{ws + bp.off_dqdyn16, false, false};
    // the tensor-core launches exist for the 16-bit I/O types only
    constexpr bool kTc = sizeof(T) == 2;
    auto tc_launch = [&](const bwd_tc::Launch& Lc) {
        if constexpr (kTc) note(bwd_tc::launch_bwd_d<T>(Lc, st));
    };
    auto tc_latent = [&](Operand A, Operand C, Operand Bc, Operand Ec, bool acc2, bool col, const float2* stt,
                         int64_t stride) {
        bwd_tc::Launch Lc = base;
        Lc.a = A; Lc.c = C; Lc.b = Bc; Lc.e = Ec; Lc.rows_tok = false; Lc.has_acc2 = acc2; Lc.stats_per_col = col;
        Lc.stats = stt; Lc.stats_stride = stride; Lc.epi = bwd_tc::kEpiPartials; Lc.part1 = part1; Lc.part2 = part2;
        tc_launch(Lc);
    };
    // SIMT operands: fp32 routing queries (the SIMT forward's) when gated
    bwd::Params sp{};
    sp.B = s.B; sp.H = s.H; sp.N = s.N; sp.M = s.M;
    sp.tok_row = pl.tok.row; sp.tok_h = pl.tok.h; sp.tok_b = pl.tok.b;
    sp.scale_log2 = pl.scale_log2; sp.scale = scale; sp.chunks = bp.chunks; sp.chunk_len = bp.chunk_len;
    sp.lse_tok = reinterpret_cast<float*>(ws + bp.off_lse_tok);
    sp.delta_tok = reinterpret_cast<float*>(ws + bp.off_delta_tok);
    sp.dk_acc = reinterpret_cast<float*>(ws + bp.off_dk_acc);
    sp.part1 = part1; sp.part2 = part2;
    sp.Zlat = z32;
    const void* q_simt = gated ? c.q_state : a.q_fixed;
    const int q_bh = gated ? s.H : 0;
    const dim3 tok_grid((unsigned)bp.tok_blocks, (unsigned)s.bh());
    const dim3 lat_grid((unsigned)bp.chunks, (unsigned)s.bh(), (unsigned)bp.row_blocks);
    constexpr int kT = bwd::kThreads;

    if (stage == 1) {
        // decode y = SDPA(k, q, z) over this rank's tokens; the latent side's
        // chunk partials reduced into region 1
        if (kTc && tcp) {
            if constexpr (kTc)
                note(tc::cp_decode<T>(tc_problem(s, pl), q_lat.ptr, !gated, z16, a.k, nullptr, st, stats_tok,
                                      bp.n_pad, a.dy));
            tc_latent(q_lat, z_lat, k, dyo, true, true, stats_tok, bp.n_pad);
        } else {
            sp.Qlat = q_simt; sp.q_batch_heads = q_bh; sp.Ktok = a.k; sp.dYtok = a.dy;
            if (gated) {
                launch(bwd::decode_rows<T, float, D>, tok_grid, dim3(kT), sp); ev.mark(st);
                launch(bwd::decode_cols<T, float, D>, lat_grid, dim3(kT), sp); ev.mark(st);
            } else {
                launch(bwd::decode_rows<T, T, D>, tok_grid, dim3(kT), sp); ev.mark(st);
                launch(bwd::decode_cols<T, T, D>, lat_grid, dim3(kT), sp); ev.mark(st);
            }
        }
        rp.part1 = part1; rp.part2 = part2; rp.chunks = bp.chunks; rp.scale = scale;
        rp.mode = bwd::kReduceDecode; rp.z = z32; rp.dz = r1z; rp.dq = r1q; rp.delta = delta_enc;
        reduce(rp);
    } else if (stage == 2) {
        // region 1 holds the summed (dq_dec, dz): dz, <dz, z> and the encode's statistics
        rp.part1 = r1q; rp.part2 = r1z; rp.chunks = 1; rp.scale = 1.f;
        rp.mode = bwd::kReduceDecode; rp.z = z32; rp.dz = dz; rp.dq = dq; rp.delta = delta_enc;
        if (tcp) { rp.out16 = ws + bp.off_dz16; rp.stats_out = stats_enc; rp.stats_stride = bp.m_pad; rp.lse_in = c.lse_enc; }
        reduce(rp);
        if (tcp) {
            bwd_tc::Launch Lc = base;
            Lc.a = k; Lc.c = dyo; Lc.c2 = v; Lc.b = q_lat; Lc.e = z_lat; Lc.e2 = dz_lat;
            Lc.dual = true; Lc.rows_tok = true; Lc.has_acc2 = true; Lc.stats_per_col = false;
            Lc.stats = stats_tok; Lc.stats_stride = bp.n_pad; Lc.stats2 = stats_enc; Lc.stats2_stride = bp.m_pad;
            Lc.epi = bwd_tc::kEpiTokDkDv; Lc.out1 = a.dk; Lc.out2 = a.dv;
            tc_launch(Lc);
            tc_latent(q_lat, dz_lat, k, v, false, false, stats_enc, bp.m_pad);
        } else {
            sp.Qlat = q_simt; sp.q_batch_heads = q_bh; sp.dOlat = dz; sp.lse_lat = c.lse_enc; sp.delta_lat = delta_enc;
            sp.Ktok = a.k; sp.Vtok = a.v; sp.dK = a.dk; sp.dV = a.dv;
            if (gated) {
                launch(bwd::token_cols<T, float, D>, tok_grid, dim3(kT), sp); ev.mark(st);
                launch(bwd::latent_rows<T, float, D>, lat_grid, dim3(kT), sp); ev.mark(st);
            } else {
                launch(bwd::token_cols<T, T, D>, tok_grid, dim3(kT), sp); ev.mark(st);
                launch(bwd::latent_rows<T, T, D>, lat_grid, dim3(kT), sp); ev.mark(st);
            }
        }
        bwd::ReduceParams r = rp;
        r.part1 = part1; r.chunks = bp.chunks; r.scale = scale; r.mode = bwd::kReduceSynthesis; r.dq0b = r2;
        r.out16 = nullptr; r.stats_out = nullptr;
        reduce(r);
    } else if (stage == 3) {
        // region 2 holds the summed dq_enc: dq, dq_dyn and the synthesis' statistics
        rp.part1 = r2; rp.chunks = 1; rp.scale = 1.f; rp.mode = bwd::kReduceEncode; rp.dq = dq;
        rp.gate = a.gate; rp.qdyn = c.qdyn; rp.dqdyn = dqdyn; rp.delta = delta0;
        if (tcp && gated) {
            rp.out16 = ws + bp.off_dqdyn16; rp.stats_out = stats_syn; rp.stats_stride = bp.m_pad; rp.lse_in = c.lse_syn;
        }
        reduce(rp);
        if (gated) {
            if (norm) {
                ev.mark(st);
                rms_norm(s, a.q0, ws + pl.off_q0n, a.k0, ws + pl.off_k0n, st);
                ev.mark(st);
            }
            if (tcp) {
                bwd_tc::Launch Lc = base;
                Lc.a = k0o; Lc.c = k0o; Lc.b = q0o; Lc.e = dqdyn_lat; Lc.rows_tok = true; Lc.has_acc2 = true;
                Lc.stats_per_col = true; Lc.stats = stats_syn; Lc.stats_stride = bp.m_pad;
                Lc.epi = bwd_tc::kEpiTokDk0; Lc.out1 = a.dk0; Lc.out2 = nullptr;
                tc_launch(Lc);
                tc_latent(q0o, dqdyn_lat, k0o, k0o, false, false, stats_syn, bp.m_pad);
            } else {
                sp.Qlat = q0s; sp.q_batch_heads = 0; sp.dOlat = dqdyn; sp.lse_lat = c.lse_syn; sp.delta_lat = delta0;
                sp.Ktok = k0s; sp.Vtok = k0s; sp.dK = a.dk0; sp.dV = nullptr;
                launch(bwd::token_cols<T, T, D>, tok_grid, dim3(kT), sp); ev.mark(st);
                launch(bwd::latent_rows<T, T, D>, lat_grid, dim3(kT), sp); ev.mark(st);
            }
            bwd::ReduceParams r{};
            r.B = s.B; r.H = s.H; r.M = s.M; r.part1 = part1; r.chunks = bp.chunks; r.scale = scale;
            r.mode = bwd::kReduceSynthesis; r.dq0b = r3;
            reduce(r);
            if (norm) {
                // dk0 (this rank's tokens) through the normalisation
                const int64_t rows_k = s.bh() * s.N;
                const int rw = 32 / (D * (int)sizeof(T) / 16);
                const int64_t want = (rows_k + 8 * rw - 1) / (8 * rw);
                bwd::rms_backward_rows_coop<T, D><<<(unsigned)std::min<int64_t>(want, (int64_t)kNumSMs * 16), 256, 0,
                                                   st>>>(static_cast<const T*>(a.k0), static_cast<T*>(a.dk0), rows_k,
                                                         kNormEps);
                ev.mark(st);
            }
        }
    } else {
        // region 3 holds the summed dq0 per batch element: the batch-shared gradients
        if (gated) {
            rp.part1 = r3; rp.chunks = 1; rp.scale = 1.f; rp.mode = bwd::kReduceSynthesis; rp.dq0b = dq0b;
            reduce(rp);
        }
        bwd::BatchParams bt{};
        bt.B = s.B; bt.H = s.H; bt.M = s.M;
        bt.dq = dq; bt.dq_fixed = a.dq_fixed;
        if (gated) { bt.dq0b = dq0b; bt.qdyn = c.qdyn; bt.dq0 = a.dq0; bt.dgate = a.dgate; }
        launch(bwd::reduce_batch<D>, dim3((unsigned)s.H), dim3(256), bt);
        ev.mark(st);
        if (norm) {
            const int64_t rows_q = (int64_t)s.H * s.M;
            bwd::rms_backward_rows<T, float, D><<<(unsigned)((rows_q + 255) / 256), 256, 0, st>>>(
                static_cast<const T*>(a.q0), a.dq0, rows_q, kNormEps);
            ev.mark(st);
        }
    }
    if (err == cudaSuccess) err = launch.err;
    if (err == cudaSuccess && cudaGetLastError() != cudaSuccess) err = cudaErrorLaunchFailure;
    return err;
}

template <typename T>
cudaError_t cp_stage_d(int stage, const Shape& s, const BwdPlan& bp, const CpBwdArgs& c, char* state,
                       StageEvents& ev, cudaStream_t st) {
    switch (s.D) {
        case 16: return cp_stage<T, 16>(stage, s, bp, c, state, ev, st);
        case 32: return cp_stage<T, 32>(stage, s, bp, c, state, ev, st);
        case 64: return cp_stage<T, 64>(stage, s, bp, c, state, ev, st);
        default: return cp_stage<T, 128>(stage, s, bp, c, state, ev, st);
    }
}

int cp_bwd_stage(int stage, const CpBwdArgs& c, void* state, int B, int H, int N, int M, int D, int dtype,
                 const flarepp_options_t* opts, void* stream) {
    const Shape s{B, H, N, M, D, dtype};
    BwdPlan bp{};
    int rc = make_bwd_plan(s, opts, &bp);
    if (rc) return rc;
    if (stage < 1 || stage > 4) return FLAREPP_ERR_INVALID_ARG;
    rc = check_bwd_pointers(s, c.a);
    if (rc) return rc;
    const bool gated = c.a.gate != nullptr;
    if (!state || reinterpret_cast<uintptr_t>(state) % kAlign || !c.z_state || !c.lse_enc ||
        (gated && (!c.q_state || !c.lse_syn || !c.qdyn)))
        return FLAREPP_ERR_INVALID_ARG;
    if (!aligned16(c.z_state) || (gated && !aligned16(c.q_state))) return FLAREPP_ERR_INVALID_ARG;
    // the CP stages take the recomputed forward's state from flarepp_cp_merge(_ex):
    // its latent inputs must keep the layout the forward's merge wrote
    if (opts && (opts->q_out || opts->z_out)) return FLAREPP_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    StageEvents ev;
    if (opts && opts->n_stage_events > 0) {
        ev.ev = opts->stage_events;
        ev.n = opts->n_stage_events;
    }
    ev.mark(st);
    char* base = static_cast<char*>(state);
    cudaError_t e;
    if (dtype == FLAREPP_F32) e = cp_stage_d<float>(stage, s, bp, c, base, ev, st);
    else if (dtype == FLAREPP_F16) e = cp_stage_d<__half>(stage, s, bp, c, base, ev, st);
    else e = cp_stage_d<__nv_bfloat16>(stage, s, bp, c, base, ev, st);
    return e == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
}

}  // namespace
}  // namespace flarepp

using namespace flarepp;

extern "C" {

int flarepp_abi_version(void) { return FLAREPP_ABI_VERSION; }

int flarepp_launches_per_call(int gated) { return gated ? 5 : 3; }

const char* flarepp_status_string(int status) {
    switch (status) {
        case FLAREPP_OK: return "ok";
        case FLAREPP_ERR_INVALID_ARG: return "invalid argument";
        case FLAREPP_ERR_UNSUPPORTED: return "unsupported shape or option";
        case FLAREPP_ERR_CUDA: return "CUDA error";
        case FLAREPP_ERR_WORKSPACE: return "workspace too small or allocation failed";
        case FLAREPP_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

int flarepp_mixer_fwd_ex(const void* q0, const void* q_fixed, const float* gate, const void* k0,
                         const void* k, const void* v, void* y, int B, int H, int N, int M, int D,
                         int dtype, const flarepp_options_t* opts, void* stream) {
    return forward(q0, q_fixed, gate, k0, k, v, y, B, H, N, M, D, dtype, opts, stream);
}

int flarepp_mixer_fwd(const void* q0, const void* q_fixed, const float* gate, const void* k0,
                      const void* k, const void* v, void* y, int B, int H, int N, int M, int D,
                      int dtype, void* stream) {
    return forward(q0, q_fixed, gate, k0, k, v, y, B, H, N, M, D, dtype, nullptr, stream);
}

int flare_fwd(const void* q, const void* k, const void* v, void* y, int B, int H, int N, int M,
              int D, int dtype, void* stream) {
    return forward(nullptr, q, nullptr, nullptr, k, v, y, B, H, N, M, D, dtype, nullptr, stream);
}

int flarepp_mixer_fwd_debug(const void* q0, const void* q_fixed, const float* gate, const void* k0,
                            const void* k, const void* v, void* y, int B, int H, int N, int M, int D,
                            int dtype, float* q_out, float* z_out, int force_chunks, void* stream) {
    if (force_chunks < 0) return FLAREPP_ERR_INVALID_ARG;
    flarepp_options_t o{};
    o.q_out = q_out;
    o.z_out = z_out;
    o.force_chunks = force_chunks;
    return forward(q0, q_fixed, gate, k0, k, v, y, B, H, N, M, D, dtype, &o, stream);
}

int flarepp_set_workspace(void* dev_ptr, size_t bytes) {
    if (dev_ptr && (reinterpret_cast<uintptr_t>(dev_ptr) % kAlign)) return FLAREPP_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FLAREPP_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_registered_mu);
    g_registered[dev].ptr = dev_ptr;
    g_registered[dev].bytes = dev_ptr ? bytes : 0;
    return FLAREPP_OK;
}

int flarepp_mixer_fwd_noalloc(const void* q0, const void* q_fixed, const float* gate, const void* k0,
                              const void* k, const void* v, void* y, int B, int H, int N, int M, int D,
                              int dtype, void* stream) {
    const Shape s{B, H, N, M, D, dtype};
    int rc = check_shape(s);
    if (rc) return rc;
    rc = check_pointers(s, q0, q_fixed, gate, k0, k, v, y);    // before any CUDA call
    if (rc) return rc;
    const int chunks = chunks_fitting_static_scratch(s);
    if (chunks < 1) return FLAREPP_ERR_WORKSPACE;   // needs more than FLAREPP_NOALLOC_SCRATCH_BYTES
    void* scratch = static_scratch_address();
    if (!scratch) return FLAREPP_ERR_CUDA;
    flarepp_options_t o{};
    o.force_chunks = chunks;
    o.workspace = scratch;
    o.workspace_bytes = kStaticScratchBytes;
    return forward(q0, q_fixed, gate, k0, k, v, y, B, H, N, M, D, dtype, &o, stream);
}

size_t flarepp_workspace_bytes(int B, int H, int N, int M, int D, int dtype, int gated,
                               const flarepp_options_t* opts) {
    (void)gated;  // the same scratch serves both forms
    const Shape s{B, H, N, M, D, dtype};
    Plan pl{};
    if (make_plan(s, opts, &pl)) return 0;
    return pl.total;
}

int flarepp_selected_path(int B, int H, int N, int M, int D, int dtype) {
    const Shape s{B, H, N, M, D, dtype};
    Plan pl{};
    if (make_plan(s, nullptr, &pl)) return 0;
    return pl.path;
}

int flarepp_selftest_wait_timeout(void* stream, unsigned int limit_us) {
    if (limit_us == 0 || limit_us > 1000000u) return FLAREPP_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    tc::wait_timeout_selftest<<<1, 32, 0, st>>>(static_cast<unsigned long long>(limit_us) * 1000ull);
    return cudaGetLastError() == cudaSuccess ? FLAREPP_OK : FLAREPP_ERR_CUDA;
}

int flarepp_check_device_status(void* stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return FLAREPP_ERR_CUDA;
    int code = 0;
    if (cudaMemcpyFromSymbol(&code, g_device_status, sizeof(int)) != cudaSuccess) return FLAREPP_ERR_CUDA;
    if (code != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return FLAREPP_ERR_CUDA;
    }
    return code;
}

size_t flarepp_cp_triple_bytes(int B, int H, int M, int D) {
    const Shape s{B, H, 1, M, D, FLAREPP_F32};
    if (check_shape(s)) return 0;
    return (size_t)s.bh() * M * (D + 2) * sizeof(float);
}

size_t flarepp_cp_latent_bytes(int B, int H, int M, int D, int dtype) {
    const Shape s{B, H, 1, M, D, dtype};
    if (check_shape(s)) return 0;
    return latent_state_bytes(s);
}

int flarepp_cp_partials(const void* q, int q_shared, const void* k, const void* v, float* triple, int B, int H,
                        int N, int M, int D, int dtype, const flarepp_options_t* opts, void* stream) {
    return cp_partials(q, q_shared, k, v, triple, B, H, N, M, D, dtype, opts, stream);
}

int flarepp_cp_merge(const float* gathered, int ranks, const void* q_fixed, const float* gate, void* state, int B,
                     int H, int M, int D, int dtype, void* stream) {
    return cp_merge(gathered, ranks, q_fixed, gate, state, B, H, M, D, dtype, stream);
}

int flarepp_cp_merge_ex(const float* gathered, int ranks, const void* q_fixed, const float* gate, void* state,
                        float* lse_out, float* pregate_out, int B, int H, int M, int D, int dtype, void* stream) {
    return cp_merge(gathered, ranks, q_fixed, gate, state, B, H, M, D, dtype, stream, lse_out, pregate_out);
}

int flarepp_cp_bwd_layout(int B, int H, int N, int M, int D, int dtype, const flarepp_options_t* opts,
                          flarepp_cp_bwd_layout_t* out) {
    const Shape s{B, H, N, M, D, dtype};
    BwdPlan bp{};
    int rc = make_bwd_plan(s, opts, &bp);
    if (rc) return rc;
    if (!out) return FLAREPP_ERR_INVALID_ARG;
    const CpLayout L = cp_layout(s, bp);
    const size_t latd = (size_t)s.bh() * M * D * sizeof(float);
    out->bytes = L.total;
    out->reduce_offset[0] = L.r1; out->reduce_bytes[0] = 2 * latd;
    out->reduce_offset[1] = L.r2; out->reduce_bytes[1] = latd;
    out->reduce_offset[2] = L.r3; out->reduce_bytes[2] = latd;
    return FLAREPP_OK;
}

int flarepp_cp_bwd_stage(int stage, const void* q0, const void* q_fixed, const float* gate, const void* q_state,
                         const void* z_state, const float* lse_syn, const float* lse_enc, const float* qdyn,
                         const void* k0, const void* k, const void* v, const void* dy, float* dq0, float* dq_fixed,
                         float* dgate, void* dk0, void* dk, void* dv, void* state, int B, int H, int N, int M, int D,
                         int dtype, const flarepp_options_t* opts, void* stream) {
    CpBwdArgs c{};
    c.a.q0 = q0; c.a.q_fixed = q_fixed; c.a.gate = gate; c.a.k0 = k0; c.a.k = k; c.a.v = v; c.a.dy = dy;
    c.a.dq0 = dq0; c.a.dq_fixed = dq_fixed; c.a.dgate = dgate; c.a.dk0 = dk0; c.a.dk = dk; c.a.dv = dv;
    c.q_state = q_state; c.z_state = z_state; c.lse_syn = lse_syn; c.lse_enc = lse_enc; c.qdyn = qdyn;
    return cp_bwd_stage(stage, c, state, B, H, N, M, D, dtype, opts, stream);
}

int flarepp_cp_decode(const void* q, int q_shared, const void* z_state, const void* k, void* y, int B, int H, int N,
                      int M, int D, int dtype, const flarepp_options_t* opts, void* stream) {
    return cp_decode(q, q_shared, z_state, k, y, B, H, N, M, D, dtype, opts, stream);
}

int flarepp_mixer_bwd(const void* q0, const void* q_fixed, const float* gate, const void* k0, const void* k,
                      const void* v, const void* dy, float* dq0, float* dq_fixed, float* dgate, void* dk0, void* dk,
                      void* dv, int B, int H, int N, int M, int D, int dtype, const flarepp_options_t* opts,
                      void* stream) {
    BwdArgs a{};
    a.q0 = q0; a.q_fixed = q_fixed; a.gate = gate; a.k0 = k0; a.k = k; a.v = v; a.dy = dy;
    a.dq0 = dq0; a.dq_fixed = dq_fixed; a.dgate = dgate; a.dk0 = dk0; a.dk = dk; a.dv = dv;
    return backward(a, B, H, N, M, D, dtype, opts, stream);
}

size_t flarepp_train_context_bytes(int B, int H, int N, int M, int D, int dtype) {
    const Shape s{B, H, N, M, D, dtype};
    if (check_shape(s)) return 0;
    return context_layout(s).total;
}

int flarepp_mixer_fwd_train(const void* q0, const void* q_fixed, const float* gate, const void* k0, const void* k,
                            const void* v, void* y, int B, int H, int N, int M, int D, int dtype,
                            const flarepp_options_t* opts, void* ctx, size_t ctx_bytes, void* stream) {
    return forward_train(q0, q_fixed, gate, k0, k, v, y, B, H, N, M, D, dtype, opts, ctx, ctx_bytes, stream);
}

int flarepp_mixer_bwd_ctx(const void* q0, const void* q_fixed, const float* gate, const void* k0, const void* k,
                          const void* v, const void* y, const void* dy, float* dq0, float* dq_fixed, float* dgate,
                          void* dk0, void* dk, void* dv, int B, int H, int N, int M, int D, int dtype,
                          const flarepp_options_t* opts, const void* ctx, size_t ctx_bytes, void* stream) {
    BwdArgs a{};
    a.q0 = q0; a.q_fixed = q_fixed; a.gate = gate; a.k0 = k0; a.k = k; a.v = v; a.dy = dy;
    a.dq0 = dq0; a.dq_fixed = dq_fixed; a.dgate = dgate; a.dk0 = dk0; a.dk = dk; a.dv = dv;
    if (!ctx) return FLAREPP_ERR_INVALID_ARG;
    return backward(a, B, H, N, M, D, dtype, opts, stream, ctx, ctx_bytes, y);
}

size_t flarepp_mixer_bwd_workspace_bytes(int B, int H, int N, int M, int D, int dtype,
                                         const flarepp_options_t* opts) {
    const Shape s{B, H, N, M, D, dtype};
    BwdPlan bp{};
    if (make_bwd_plan(s, opts, &bp)) return 0;
    return bp.total;
}

int flarepp_mixer_bwd_launches(int gated, int path) {
    if (path == FLAREPP_PATH_TCGEN05) return gated ? 5 + 9 : 3 + 6;
    return gated ? 4 + 10 : 2 + 7;
}

int flarepp_mixer_fwd_host(const void* q0, const void* q_fixed, const float* gate, const void* k0,
                           const void* k, const void* v, void* y, int B, int H, int N, int M, int D,
                           int dtype, void* stream) {
    return host_forward(q0, q_fixed, gate, k0, k, v, y, B, H, N, M, D, dtype, stream);
}

}  // extern "C"
