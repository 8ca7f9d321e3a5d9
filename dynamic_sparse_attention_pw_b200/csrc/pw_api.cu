// pw_api.cu -- the extern "C" entry points declared in include/pw.h: argument checks on the
// host, workspace carving, and the kernel launches of pw_group.cu and pw_attn.cu.
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "pw_internal.h"

namespace {

using namespace pw;

struct Sizes {
    int64_t T = 0, n_windows = 0, n_groups = 0, union_cap = 0;
    int32_t words = 0;
};

constexpr size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

pw_status compute_sizes(const int32_t *cu_host, int B, int Hkv, int kmax, int W, int g, Sizes &z)
{
    if (!cu_host || B < 1 || Hkv < 1 || kmax < 1 || W < 1 || g < 1)
        return PW_ERR_INVALID_ARG;
    if (cu_host[0] != 0)
        return PW_ERR_INVALID_ARG;
    if (g > kMaxGroupSize || W > kMaxWindow || W % g != 0 || kmax > 0xFFFF)
        return PW_ERR_UNSUPPORTED;
    int maxp = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t len = static_cast<int64_t>(cu_host[b + 1]) - cu_host[b];
        if (len < 0)
            return PW_ERR_INVALID_ARG;
        const int64_t P = (len + kPageTokens - 1) / kPageTokens;
        if (P > 32 * kMaxWords)
            return PW_ERR_UNSUPPORTED;
        if (P > maxp)
            maxp = static_cast<int>(P);
        const int64_t nwin = (len + W - 1) / W;
        const int64_t gpb = (len / W) * (W / g) + ((len % W) + g - 1) / g;
        z.n_windows += nwin * Hkv;
        z.n_groups += gpb * Hkv;
        const int64_t per = static_cast<int64_t>(g) * kmax < P ? static_cast<int64_t>(g) * kmax : P;
        z.union_cap += gpb * Hkv * per;
    }
    z.T = cu_host[B];
    z.words = (maxp + 31) / 32;
    if (z.words < 1)
        z.words = 1;
    if (z.union_cap >= (static_cast<int64_t>(1) << 31) || z.n_groups >= (static_cast<int64_t>(1) << 31))
        return PW_ERR_UNSUPPORTED;
    return PW_OK;
}

size_t workspace_for(const Sizes &z, int Hkv)
{
    size_t ws = 0;
    ws += align256(static_cast<size_t>(z.T) * Hkv * sizeof(uint16_t)); // set sizes
    ws += align256(static_cast<size_t>(z.n_groups) * sizeof(int32_t));  // union sizes
    ws += align256(static_cast<size_t>(z.n_groups) * z.words * sizeof(uint32_t)); // union bitsets
    return ws < 256 ? 256 : ws;
}

} // namespace

extern "C" {

int pw_version(void) { return 101; }

const char *pw_status_string(int s)
{
    switch (s) {
    case PW_OK: return "ok";
    case PW_ERR_INVALID_ARG: return "invalid argument";
    case PW_ERR_UNSUPPORTED: return "unsupported shape";
    case PW_ERR_BAD_SELECTION: return "selected page outside the query's causal prefix";
    case PW_ERR_CAPACITY: return "buffer smaller than required";
    case PW_ERR_TIMEOUT: return "bounded device wait ran out";
    case PW_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
    }
}

pw_status pw_groups_size(const int32_t *cu_seqlens_host, int B, int Hkv, int kmax, int W, int g,
                         int64_t *n_groups, int64_t *union_cap, int32_t *words,
                         size_t *workspace_bytes)
{
    Sizes z;
    const pw_status st = compute_sizes(cu_seqlens_host, B, Hkv, kmax, W, g, z);
    if (st != PW_OK)
        return st;
    if (n_groups)
        *n_groups = z.n_groups;
    if (union_cap)
        *union_cap = z.union_cap;
    if (words)
        *words = z.words;
    if (workspace_bytes)
        *workspace_bytes = workspace_for(z, Hkv);
    return PW_OK;
}

pw_status pw_group(const int32_t *sel_pages, const int32_t *cu_seqlens,
                   const int32_t *cu_seqlens_host, int B, int Hkv, int kmax, int W, int g,
                   const pw_groups *groups, void *workspace, size_t workspace_bytes,
                   int32_t *dev_status, void *stream)
{
    Sizes z;
    pw_status st = compute_sizes(cu_seqlens_host, B, Hkv, kmax, W, g, z);
    if (st != PW_OK)
        return st;
    if (!groups || !cu_seqlens || !dev_status || (z.T > 0 && !sel_pages))
        return PW_ERR_INVALID_ARG;
    if (groups->g != g || groups->words != z.words || groups->n_groups != z.n_groups)
        return PW_ERR_INVALID_ARG;
    if (groups->union_cap < z.union_cap || workspace_bytes < workspace_for(z, Hkv) || !workspace)
        return PW_ERR_CAPACITY;
    if (!groups->union_off || !groups->bits ||
        (z.n_groups > 0 && (!groups->qids || !groups->gsize || !groups->gmeta)) ||
        (z.union_cap > 0 && !groups->union_pages))
        return PW_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return PW_ERR_INVALID_ARG;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess)
        return PW_ERR_CUDA;

    uint8_t *w = static_cast<uint8_t *>(workspace);
    GroupLaunch L{};
    L.sel = sel_pages;
    L.cu = cu_seqlens;
    L.B = B;
    L.Hkv = Hkv;
    L.kmax = kmax;
    L.W = W;
    L.g = g;
    L.words = z.words;
    L.T = z.T;
    L.n_windows = z.n_windows;
    L.n_groups = z.n_groups;
    L.union_cap = groups->union_cap;
    L.bits = groups->bits;
    L.counts = reinterpret_cast<uint16_t *>(w);
    w += align256(static_cast<size_t>(z.T) * Hkv * sizeof(uint16_t));
    L.ucount = reinterpret_cast<int32_t *>(w);
    w += align256(static_cast<size_t>(z.n_groups) * sizeof(int32_t));
    L.ubits = reinterpret_cast<uint32_t *>(w);
    L.qids = groups->qids;
    L.gsize = groups->gsize;
    L.gmeta = groups->gmeta;
    L.union_off = groups->union_off;
    L.union_pages = groups->union_pages;
    L.status = dev_status;
    return group_launch(L, s) == cudaSuccess ? PW_OK : PW_ERR_CUDA;
}

pw_status pw_attn(const void *Q, const void *K_pages, const void *V_pages,
                  const int32_t *page_table, int max_pages, int n_phys,
                  const int32_t *cu_seqlens, int B, int64_t T, int Hq, int Hkv,
                  float k_scale, float v_scale, float sm_scale,
                  const pw_groups *groups, void *O, int32_t *dev_status, void *stream)
{
    if (!groups || !cu_seqlens || !dev_status || B < 1 || T < 0 || Hq < 1 || Hkv < 1 ||
        max_pages < 0 || n_phys < 0)
        return PW_ERR_INVALID_ARG;
    if (Hq % Hkv != 0)
        return PW_ERR_UNSUPPORTED;
    const int G = Hq / Hkv;
    if (groups->g < 1 || groups->g > kMaxGroupSize || groups->g * G > kMaxTileRows)
        return PW_ERR_UNSUPPORTED;
    if (groups->n_groups < 0 || groups->words < 1)
        return PW_ERR_INVALID_ARG;
    if (groups->n_groups > 0 &&
        (!Q || !K_pages || !V_pages || !page_table || !O || !groups->qids || !groups->gsize ||
         !groups->gmeta || !groups->union_off || !groups->bits || !groups->sched))
        return PW_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K_pages) |
         reinterpret_cast<uintptr_t>(V_pages) | reinterpret_cast<uintptr_t>(O)) & 15u)
        return PW_ERR_INVALID_ARG;
    AttnLaunch L{};
    L.Q = static_cast<const uint16_t *>(Q);
    L.K = static_cast<const uint8_t *>(K_pages);
    L.V = static_cast<const uint8_t *>(V_pages);
    L.page_table = page_table;
    L.max_pages = max_pages;
    L.n_phys = n_phys;
    L.cu = cu_seqlens;
    L.B = B;
    L.Hq = Hq;
    L.Hkv = Hkv;
    L.G = G;
    L.T = T;
    L.k_scale = k_scale;
    L.v_scale = v_scale;
    L.sm_scale = sm_scale;
    L.qids = groups->qids;
    L.gsize = groups->gsize;
    L.gmeta = groups->gmeta;
    L.union_off = groups->union_off;
    L.union_pages = groups->union_pages;
    L.bits = groups->bits;
    L.sched = groups->sched;
    L.dyn_sched = B > 1 ? 1 : 0;
    L.words = groups->words;
    L.g = groups->g;
    L.n_groups = groups->n_groups;
    L.O = static_cast<uint16_t *>(O);
    L.status = dev_status;
    return attn_launch(L, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PW_OK : PW_ERR_CUDA;
}

} // extern "C"
