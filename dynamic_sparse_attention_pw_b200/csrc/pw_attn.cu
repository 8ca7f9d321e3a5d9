// pw_attn.cu -- ID-aware union attention of PageWeaver on sm_100a.
//
// "PageWeaver: KV-Guided Query Unions for Sparse Attention" (arXiv 2610.11201), Abstract:
// query unions share page loads and populate tensor-core tiles; each query keeps its original
// support and complete output ownership; the kernel consumes query IDs without materialising
// reordered Q tensors or cross-page partial outputs; FP8 KV throughout.
//
// One CTA (4 warps) owns one group.  Tile row r = member * G + head (G = Hq / Hkv query heads
// share the member's kv head and selection), rows >= gsize * G are padding.  Per union page,
// in ascending order:
//   bulk copy   K and V page (E4M3, 8 KiB each) via the page table into a 2-stage ring
//   decode      E4M3 -> f16 (exact) into 128-byte-swizzled operand tiles
//   S = Q K^T   tcgen05.mma kind::f16, M=128, N=64, K=128 -> TMEM (fp32)
//   mask        row keeps page p only if p is in its token's own selection, and keys <= its
//               position (causal limit on the own page)
//   softmax     online, fp32, base 2; the running max is raised lazily (only when it grows by
//               more than 2^8) so the O rescale in TMEM is rare; P is split into f16 hi + lo
//   O += P V    two tcgen05.mma (P_hi V, P_lo V), M=128, N=128, K=64 -> TMEM (fp32)
// Epilogue: O / l, times v_scale, round to bf16, each row written to its own O[t, hq, :].
//
// Numerics: K and V are exact in f16 (E4M3 is a subset).  Q (bf16) is scaled per row by a
// power of two into f16's range, which is exact for every element within 2^-25 of the row
// maximum; the power of two is folded into the row's score scale.  The hi + lo split carries
// P with about 22 significant bits into the fp32 PV accumulation.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "pw_internal.h"
#include "pw_sm100.cuh"

namespace pw {
namespace {

constexpr int kThreads = 128;
constexpr int kStages = 2;
constexpr int kPageBytes = kPageTokens * kHeadDim; // one kv head's page, E4M3
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;   // S: 64 fp32 columns
constexpr uint32_t kColO = 128; // O: 128 fp32 columns
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kIdescS = idesc_f16_f32(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_f16_f32(128, 128, false, true);

// Operand tiles.  q: [2 dim-blocks][128 rows][128 B]; k and v: [2 dim-blocks][64 keys][128 B];
// p: [128 rows][128 B].  Rows are 128 bytes (64 f16), 16-byte chunks XOR-swizzled by row % 8,
// 8-row atoms at 1024 bytes.  The same physical layout serves K as the K-major B operand of
// S = Q K^T and V as the MN-major B operand of O = P V.
struct __align__(1024) AttnSmem {
    uint8_t q[2][128 * 128];
    uint8_t k[2][64 * 128];
    uint8_t v[2][64 * 128];
    uint8_t p_hi[128 * 128];
    uint8_t p_lo[128 * 128];
    uint8_t stage_k[kStages][kPageBytes];
    uint8_t stage_v[kStages][kPageBytes];
    uint64_t tma_bar[kStages];
    uint64_t mma_bar;
    uint32_t tmem_base;
};

constexpr size_t kSmemBytes = sizeof(AttnSmem) + 1024;

__device__ __forceinline__ uint32_t swz(int row, int chunk)
{
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes)
{
    const __half2_raw h =
        __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xFFFFu), __NV_E4M3);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// 64 keys x 128 dims E4M3 (row-major) -> two swizzled 64-dim f16 blocks.
__device__ __forceinline__ void decode_page(const uint8_t *src, uint8_t (*dst)[64 * 128], int tid)
{
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
        const int q = tid + kThreads * rep;
        const int row = q >> 3, c16 = q & 7;
        const uint4 x = *reinterpret_cast<const uint4 *>(src + row * 128 + c16 * 16);
        uint4 h0, h1;
        h0.x = e4m3x2_to_f16x2(x.x);
        h0.y = e4m3x2_to_f16x2(x.x >> 16);
        h0.z = e4m3x2_to_f16x2(x.y);
        h0.w = e4m3x2_to_f16x2(x.y >> 16);
        h1.x = e4m3x2_to_f16x2(x.z);
        h1.y = e4m3x2_to_f16x2(x.z >> 16);
        h1.z = e4m3x2_to_f16x2(x.w);
        h1.w = e4m3x2_to_f16x2(x.w >> 16);
        uint8_t *blk = dst[c16 >> 2];
        const int j0 = (2 * c16) & 7;
        *reinterpret_cast<uint4 *>(blk + swz(row, j0)) = h0;
        *reinterpret_cast<uint4 *>(blk + swz(row, j0 + 1)) = h1;
    }
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_h2(__half a, __half b)
{
    return static_cast<uint32_t>(__half_as_ushort(a)) |
           (static_cast<uint32_t>(__half_as_ushort(b)) << 16);
}

__global__ void __launch_bounds__(kThreads, 1) k_union_attn(const AttnLaunch L)
{
    extern __shared__ uint8_t smem_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t gi = blockIdx.x;

    const int b = L.gmeta[3 * gi + 0];
    const int h = L.gmeta[3 * gi + 1];
    const int R = L.gsize[gi] * L.G;
    const int u0 = L.union_off[gi];
    const int nU = L.union_off[gi + 1] - u0;

    // Once any CTA of this launch has given up on a wait, the rest skip their work instead of
    // each waiting out its own limit.
    if (tid == 0)
        sm.tmem_base = *reinterpret_cast<volatile int32_t *>(L.status) == PW_ERR_TIMEOUT ? 1u : 0u;
    __syncthreads();
    if (sm.tmem_base != 0u)
        return;
    __syncthreads();

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s)
            mbar_init(&sm.tma_bar[s], 1);
        mbar_init(&sm.mma_bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }

    // ---- row metadata and the Q tile (row r = thread r = TMEM lane r) ----
    const int r = tid;
    const bool valid = r < R;
    int64_t t = 0;
    int hq = 0, pos = 0, own = 0;
    const uint32_t *bitrow = nullptr;
    if (valid) {
        const int mi = r / L.G, j = r - mi * L.G;
        t = L.qids[gi * L.g + mi];
        hq = h * L.G + j;
        pos = static_cast<int>(t - L.cu[b]);
        own = pos >> 6;
        bitrow = L.bits + (static_cast<size_t>(t) * L.Hkv + h) * L.words;
    }
    float crow;
    {
        uint4 qv[16];
        const uint4 *src = reinterpret_cast<const uint4 *>(
            L.Q + (static_cast<size_t>(t) * L.Hq + hq) * kHeadDim);
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            qv[i] = valid ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                amax = fmaxf(amax, fabsf(__uint_as_float(w[e] << 16)));
                amax = fmaxf(amax, fabsf(__uint_as_float(w[e] & 0xFFFF0000u)));
            }
        }
        int s = 0;
        if (amax > 0.f && amax <= 3.0e38f) {
            int e2;
            frexpf(amax, &e2); // amax in [2^(e2-1), 2^e2)
            s = 15 - e2;       // amax * 2^s in [2^14, 2^15)
            s = s < -126 ? -126 : (s > 126 ? 126 : s);
        }
        const float up = __uint_as_float(static_cast<uint32_t>(127 + s) << 23);
        const float down = __uint_as_float(static_cast<uint32_t>(127 - s) << 23);
        crow = L.sm_scale * L.k_scale * kLog2e * down;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t w[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __half lo = __float2half_rn(__uint_as_float(w[e] << 16) * up);
                const __half hi = __float2half_rn(__uint_as_float(w[e] & 0xFFFF0000u) * up);
                o[e] = pack_h2(lo, hi);
            }
            *reinterpret_cast<uint4 *>(sm.q[i >> 3] + swz(r, i & 7)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

    auto issue_page = [&](int i, int s) {
        const int pg = L.union_pages[u0 + i];
        int phys = L.page_table[static_cast<size_t>(b) * L.max_pages + pg];
        if (phys < 0 || phys >= L.n_phys) {
            set_status(L.status, PW_ERR_INVALID_ARG);
            phys = 0;
        }
        const size_t off = (static_cast<size_t>(phys) * L.Hkv + h) * kPageBytes;
        mbar_arrive_expect_tx(&sm.tma_bar[s], 2 * kPageBytes);
        bulk_g2s(sm.stage_k[s], L.K + off, kPageBytes, &sm.tma_bar[s]);
        bulk_g2s(sm.stage_v[s], L.V + off, kPageBytes, &sm.tma_bar[s]);
    };

    if (tid == 0)
        for (int i = 0; i < kStages && i < nU; ++i)
            issue_page(i, i);

    float m_used = -INFINITY, l = 0.f;
    uint32_t mma_phase = 0;
    bool aborted = false;
    int pages_waited = 0;   // TMA phases consumed
    bool mma_pending = false;

    for (int i = 0; i < nU; ++i) {
        const int s = i % kStages;
        const int pg = L.union_pages[u0 + i];
        bool ok = true;
        if (mma_pending) { // previous O += P V: frees v, p_hi, p_lo and settles O
            ok = mbar_wait(&sm.mma_bar, mma_phase);
            mma_phase ^= 1u;
            mma_pending = false;
        }
        ok = ok && mbar_wait(&sm.tma_bar[s], static_cast<uint32_t>((i / kStages) & 1));
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        pages_waited = i + 1;
        tc_fence_after();
        decode_page(sm.stage_k[s], sm.k, tid);
        decode_page(sm.stage_v[s], sm.v, tid);
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {
            if (i + kStages < nU)
                issue_page(i + kStages, s);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t ad = sdesc_sw128(smem_u32(sm.q[kk >> 2]) + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(smem_u32(sm.k[kk >> 2]) + (kk & 3) * 32, 16, 1024);
                mma_f16_ss(tmem + kColS, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
            }
            mma_commit(&sm.mma_bar);
        }
        ok = mbar_wait(&sm.mma_bar, mma_phase);
        mma_phase ^= 1u;
        tc_fence_after();

        uint32_t sa[32], sb[32];
        tmem_ld32(tmem + lane_base + kColS, sa);
        tmem_ld32(tmem + lane_base + kColS + 32, sb);
        tmem_ld_wait(sa);
        tmem_ld_wait(sb);

        int n_allow = 0;
        if (valid) {
            const uint32_t word = __ldg(bitrow + (pg >> 5));
            if ((word >> (pg & 31)) & 1u)
                n_allow = pg < own ? 64 : (pg == own ? (pos & 63) + 1 : 0);
        }
        float x[64];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            x[j] = __uint_as_float(sa[j]) * crow;
            x[j + 32] = __uint_as_float(sb[j]) * crow;
        }
        float alpha = 1.f;
        bool rescale = false;
        if (n_allow > 0) {
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; ++j)
                if (j < n_allow)
                    mx = fmaxf(mx, x[j]);
            if (mx > m_used + kRescaleLog2) {
                if (m_used != -INFINITY) {
                    alpha = ex2(m_used - mx);
                    rescale = true;
                    l *= alpha;
                }
                m_used = mx;
            }
        }
        // P = 2^(x - m) on allowed keys, split into f16 hi + lo, written as the A operand
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = 8 * c + 2 * e;
                const float p0 = j < n_allow ? ex2(x[j] - m_used) : 0.f;
                const float p1 = j + 1 < n_allow ? ex2(x[j + 1] - m_used) : 0.f;
                l += p0 + p1;
                const __half h0 = __float2half_rn(p0), h1 = __float2half_rn(p1);
                hi[e] = pack_h2(h0, h1);
                lo[e] = pack_h2(__float2half_rn(p0 - __half2float(h0)),
                                __float2half_rn(p1 - __half2float(h1)));
            }
            *reinterpret_cast<uint4 *>(sm.p_hi + swz(r, c)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(sm.p_lo + swz(r, c)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + kColO + 32 * q, o);
                tmem_ld_wait(o);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                tmem_st32(tmem + lane_base + kColO + 32 * q, o);
            }
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = sdesc_sw128(smem_u32(sm.v) + kk * 2048, 8192, 1024);
                mma_f16_ss(tmem + kColO, sdesc_sw128(smem_u32(sm.p_hi) + kk * 32, 16, 1024), bd,
                           kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                mma_f16_ss(tmem + kColO, sdesc_sw128(smem_u32(sm.p_lo) + kk * 32, 16, 1024), bd,
                           kIdescPV, 1u);
            }
            mma_commit(&sm.mma_bar);
        }
        mma_pending = true;
    }

    bool ok = true;
    if (!aborted && mma_pending) {
        ok = mbar_wait(&sm.mma_bar, mma_phase);
        mma_phase ^= 1u;
        mma_pending = false;
    }
    if (__syncthreads_or(!ok))
        aborted = true;

    if (aborted) {
        // Drain what this CTA still has in flight (bounded), so nothing lands after exit.
        set_status(L.status, PW_ERR_TIMEOUT);
        if (tid == 0) {
            const int issued = nU < pages_waited + kStages ? nU : pages_waited + kStages;
            for (int i = pages_waited; i < issued; ++i)
                (void)mbar_wait(&sm.tma_bar[i % kStages], static_cast<uint32_t>((i / kStages) & 1));
            if (mma_pending)
                (void)mbar_wait(&sm.mma_bar, mma_phase);
        }
    } else {
        tc_fence_after();
        const float inv = (nU > 0 && l > 0.f) ? L.v_scale / l : 0.f;
        uint16_t *dst = L.O + (static_cast<size_t>(t) * L.Hq + hq) * kHeadDim;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + kColO + 32 * q, o);
            tmem_ld_wait(o);
            if (valid) {
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float a = nU > 0 ? __uint_as_float(o[2 * j]) * inv : 0.f;
                    const float c = nU > 0 ? __uint_as_float(o[2 * j + 1]) * inv : 0.f;
                    const __nv_bfloat162 v2 = __floats2bfloat162_rn(a, c);
                    pk[j] = *reinterpret_cast<const uint32_t *>(&v2);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4 *>(dst + 32 * q + 8 * j) =
                        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

} // namespace

cudaError_t attn_launch(const AttnLaunch &L, cudaStream_t st)
{
    if (L.n_groups == 0)
        return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k_union_attn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess)
        return e;
    const unsigned grid = static_cast<unsigned>(L.n_groups);
    k_union_attn<<<grid, kThreads, kSmemBytes, st>>>(L);
    return cudaGetLastError();
}

} // namespace pw
