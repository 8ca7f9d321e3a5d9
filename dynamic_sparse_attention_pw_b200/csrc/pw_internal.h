// pw_internal.h -- launch descriptors shared by the C entry points (pw_api.cu) and the
// kernel files.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/pw.h"

namespace pw {

constexpr int kPageTokens = 64;
constexpr int kHeadDim = 128;
constexpr int kMaxWindow = 256;
constexpr int kMaxWords = 64;   // sequences up to 131072 tokens
constexpr int kMaxGroupSize = 32;
constexpr int kMaxTileRows = 128;

struct GroupLaunch {
    const int32_t *sel;
    const int32_t *cu;
    int B, Hkv, kmax, W, g, words;
    int64_t T, n_windows, n_groups, union_cap;
    uint32_t *bits;
    uint16_t *counts;
    uint32_t *ubits;
    int32_t *ucount;
    int32_t *qids, *gsize, *gmeta, *union_off, *union_pages;
    int32_t *status;
};

struct AttnLaunch {
    const uint16_t *Q;      // bf16 bits
    const uint8_t *K, *V;   // E4M3 codes
    const int32_t *page_table;
    int max_pages, n_phys;
    const int32_t *cu;
    int B, Hq, Hkv, G;
    int64_t T;
    float k_scale, v_scale, sm_scale;
    const int32_t *qids, *gsize, *gmeta, *union_off, *union_pages;
    const uint32_t *bits;
    int32_t *sched;         // work counter of the persistent kernel, zeroed before its launch
    int dyn_sched;          // take groups from sched (ragged batches) instead of a fixed stride
    int words, g;
    int64_t n_groups;
    uint16_t *O;            // bf16 bits
    int32_t *status;
};

cudaError_t group_launch(const GroupLaunch &L, cudaStream_t st);
cudaError_t attn_launch(const AttnLaunch &L, cudaStream_t st);
cudaError_t attn_ws_launch(const AttnLaunch &L, cudaStream_t st); // tiles of <= 64 rows

} // namespace pw
