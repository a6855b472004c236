// tcgen05 (5th-generation tensor core) kernels of the FLARE++ mixer.
#pragma once

#include "common.cuh"

namespace flarepp {
namespace tc {

constexpr int kTokTile = 128;        // tokens per K/V tile
constexpr int kPartsPerChunk = 2;    // partial triples written per token chunk

struct Buffers {
    float* part_O;
    float2* part_ml;
    float* q32;
    __nv_bfloat16* q16;
    float* z32;
    __nv_bfloat16* z16;
};

struct Problem {
    int B, H, N, M, D;
    int chunks, chunk_len;
    float scale_log2;
};

inline bool supported(bool bf16, int D, int M) { (void)bf16; (void)D; (void)M; return false; }
inline int row_groups(int M) { return (M + 255) / 256; }
inline int target_ctas() { return 4 * kNumSMs; }

template <typename Mark>
inline int run(const Problem&, const Buffers&, const void*, const void*, const float*, const void*,
               const void*, const void*, void*, float*, float*, Mark&&, cudaStream_t) {
    return 2;  // FLAREPP_ERR_UNSUPPORTED
}

}  // namespace tc
}  // namespace flarepp
