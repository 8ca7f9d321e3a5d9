// pw_attn.cu -- ID-aware union attention of PageWeaver on sm_100a.
//
// "PageWeaver: KV-Guided Query Unions for Sparse Attention" (arXiv 2610.11201), Abstract:
// query unions share page loads and populate tensor-core tiles; each query keeps its original
// support and complete output ownership; the kernel consumes query IDs without materialising
// reordered Q tensors or cross-page partial outputs; FP8 KV throughout.
//
// One CTA owns one group.  Tile row i = member * G + head (the G = Hq / Hkv query heads share
// the member's kv head and selection); rows >= R = gsize * G are padding.  Rows are processed
// in blocks of 64 (RB blocks, 128 * RB threads).  Per union page, in ascending order:
//   bulk copy  K and V page (E4M3, 8 KiB each) via the page table into a 2-stage ring
//   decode     E4M3 -> bf16, exact, with integer bit operations (no conversion unit) into
//              128-byte-swizzled operand tiles
//   S = Q K^T  tcgen05.mma kind::f16 (bf16), M=64 per row block, N=64 keys, K=128 -> TMEM
//   mask       a row keeps page p only if p is in its own token's selection, and keys at or
//              before its position (causal limit on its own page)
//   softmax    online, fp32, base 2, two threads per row (columns 0-31 / 32-63); the running
//              max is raised lazily (only when it grows by more than 2^8) so the rescale of
//              the accumulator is rare; P is split into bf16 hi + lo with integer rounding
//   O^T += V^T P^T   tcgen05.mma M=128 (head dim), N=R rounded up to 16, K=64 keys, twice
//              (P_hi, P_lo), fp32 in TMEM -- the head dimension fills the 128 MMA rows, so no
//              MMA row is padding
// Epilogue: O / l, times v_scale, rounded to bf16, each row written to its own O[t, hq, :].
//
// Numerics: Q (bf16), K and V (E4M3 is a subset of bf16) enter the tensor cores exactly;
// products accumulate in fp32.  P = hi + lo carries about 16 significant bits (hi rounded to
// nearest, the remainder truncated), which keeps the output within the 1e-3 rel-L2 bar with a
// margin of about ten.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pw_internal.h"
#include "pw_attn_common.cuh"
#include "pw_sm100.cuh"

namespace pw {
namespace {

using namespace attn;

constexpr int kStages = 2;
constexpr uint32_t kIdescS = idesc_bf16_f32(64, 64, false, false);
constexpr int kUnionCache = 512; // union pages whose ids are staged in shared memory

// Operand tiles (rows of 128 bytes = 64 bf16, 16-byte chunks XOR-swizzled by row % 8, 8-row
// atoms at 1024 bytes):
//   q    [2 dim-blocks][RB*64 rows][128 B]  A of S (K-major); row block rb at row 64 rb
//   k    [2 dim-blocks][64 keys][128 B]     B of S (K-major)
//   v    [2 dim-blocks][64 keys][128 B]     A of O^T, read MN-major (head dim along M)
//   p_*  [RB*64 rows][128 B]                B of O^T (K-major: 64 keys per row)
template <int RB>
struct __align__(1024) AttnSmem {
    uint8_t q[2][RB * 64 * 128];
    uint8_t k[2][64 * 128];
    uint8_t v[2][64 * 128];
    uint8_t p_hi[RB * 64 * 128];
    uint8_t p_lo[RB * 64 * 128];
    uint8_t stage_k[kStages][kPageBytes];
    uint8_t stage_v[kStages][kPageBytes];
    float alpha[RB * 64];
    float inv_l[RB * 64];
    int32_t row_tok[RB * 64];
    int32_t row_hq[RB * 64];
    int32_t upage[kUnionCache]; // the group's union pages (logical), first kUnionCache
    int32_t uphys[kUnionCache]; // and their physical slots
    uint64_t tma_bar[kStages];
    uint64_t mma_bar;
    uint32_t tmem_base;
    int32_t flag;
    int32_t rescale; // some row raised its running max on this page
};

template <int RB>
__global__ void __launch_bounds__(128 * RB, (RB == 1) ? 2 : 1) k_union_attn(const AttnLaunch L)
{
    constexpr int NT = 128 * RB;
    constexpr uint32_t kColS = 0;          // S: RB blocks of 64 fp32 columns
    constexpr uint32_t kColO = 64 * RB;    // O^T: up to 64 * RB fp32 columns
    constexpr uint32_t kTmemCols = 128 * RB;
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<RB> &sm = *reinterpret_cast<AttnSmem<RB> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t gi = blockIdx.x;

    // Once any CTA of this launch has given up on a wait, the rest skip their work.
    if (tid == 0)
        sm.flag = *reinterpret_cast<volatile int32_t *>(L.status) == PW_ERR_TIMEOUT ? 1 : 0;
    __syncthreads();
    if (sm.flag != 0)
        return;

    const int b = L.gmeta[3 * gi + 0];
    const int h = L.gmeta[3 * gi + 1];
    const int R = L.gsize[gi] * L.G;
    const int Npad = (R + 15) & ~15;
    const int u0 = L.union_off[gi];
    const int nU = L.union_off[gi + 1] - u0;
    const uint32_t kIdescPV = idesc_bf16_f32(128, Npad, true, false);
    if (!group_scalars_ok(L, b, h, L.gsize[gi], nU))
        return;
    const int32_t cu_b = L.cu[b], cu_e = L.cu[b + 1];

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
    // per-row metadata
    for (int i = tid; i < 64 * RB; i += NT) {
        int32_t tok = 0, hq = 0;
        if (i < R) {
            const int mi = i / L.G;
            tok = L.qids[gi * L.g + mi];
            hq = h * L.G + (i - mi * L.G);
            if (tok < cu_b || tok >= cu_e) { // a member outside the group's sequence
                set_status(L.status, PW_ERR_INVALID_ARG);
                tok = cu_b;
            }
        }
        sm.row_tok[i] = tok;
        sm.row_hq[i] = hq;
        sm.alpha[i] = 1.f;
    }
    for (int i = tid; i < nU && i < kUnionCache; i += NT) {
        const int pg = L.union_pages[u0 + i];
        sm.upage[i] = pg;
        sm.uphys[i] = phys_page(L, b, pg);
    }
    if (tid == 0)
        sm.rescale = 0;
    __syncthreads();
    // Q tile: RB*64 rows x 16 chunks of 8 bf16, copied as is (rows >= R are zero)
    for (int qn = tid; qn < RB * 64 * 16; qn += NT) {
        const int row = qn >> 4, c = qn & 15;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (row < R)
            val = __ldg(reinterpret_cast<const uint4 *>(
                      L.Q + (static_cast<size_t>(sm.row_tok[row]) * L.Hq + sm.row_hq[row]) * kHeadDim) +
                  c);
        *reinterpret_cast<uint4 *>(sm.q[c >> 3] + swz(row, c & 7)) = val;
    }

    // Softmax role: row i = 64 rb + 16 qd + (lane % 16), key half hh = lane / 16.
    const int rb = warp >> 2, qd = warp & 3;
    const int my_row = 64 * rb + 16 * qd + (lane & 15);
    const int hh = lane >> 4;
    const bool row_valid = my_row < R;
    int pos = 0, own = 0;
    const uint32_t *bitrow = nullptr;
    if (row_valid) {
        const int64_t tok = sm.row_tok[my_row];
        pos = static_cast<int>(tok - L.cu[b]);
        own = pos >> 6;
        bitrow = L.bits + (static_cast<size_t>(tok) * L.Hkv + h) * L.words;
    }
    const float crow = L.sm_scale * L.k_scale * kLog2e;

    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t s_addr = tmem + (static_cast<uint32_t>(32 * qd) << 16) + kColS + 64 * rb;

    auto page_of = [&](int i) -> int {
        return i < kUnionCache ? sm.upage[i] : L.union_pages[u0 + i];
    };
    auto issue_page = [&](int i, int s) {
        int phys;
        if (i < kUnionCache) {
            phys = sm.uphys[i];
        } else {
            phys = phys_page(L, b, L.union_pages[u0 + i]);
        }
        const size_t off = (static_cast<size_t>(phys) * L.Hkv + h) * kPageBytes;
        mbar_arrive_expect_tx(&sm.tma_bar[s], 2 * kPageBytes);
        bulk_g2s(sm.stage_k[s], L.K + off, kPageBytes, &sm.tma_bar[s]);
        bulk_g2s(sm.stage_v[s], L.V + off, kPageBytes, &sm.tma_bar[s]);
    };
    if (tid == 0)
        for (int i = 0; i < kStages && i < nU; ++i)
            issue_page(i, i);

    float m_used = -INFINITY, l_part = 0.f;
    uint32_t mma_phase = 0;
    bool aborted = false, mma_pending = false;
    int pages_waited = 0;

    for (int i = 0; i < nU; ++i) {
        const int s = i % kStages;
        const int pg = page_of(i);
        // membership word of my row for this page, fetched now so the decode hides its latency
        const uint32_t word = row_valid ? __ldg(bitrow + page_word(L, pg)) : 0u;
        bool ok = true;
        if (mma_pending) { // previous O^T += V^T P^T: frees v and p, settles O^T
            ok = mbar_wait(&sm.mma_bar, mma_phase);
            if (ok) {
                mma_phase ^= 1u;
                mma_pending = false;
            }
        }
        ok = ok && mbar_wait(&sm.tma_bar[s], static_cast<uint32_t>((i / kStages) & 1));
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        pages_waited = i + 1;
        decode_page<NT>(sm.stage_k[s], sm.k, tid);
        decode_page<NT>(sm.stage_v[s], sm.v, tid);
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int r = 0; r < RB; ++r)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = sdesc_sw128(
                        smem_u32(sm.q[kk >> 2]) + r * 64 * 128 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(smem_u32(sm.k[kk >> 2]) + (kk & 3) * 32, 16, 1024);
                    mma_f16_ss(tmem + kColS + 64 * r, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
                }
            mma_commit(&sm.mma_bar);
            if (i + kStages < nU) // the stage was consumed by the decode above
                issue_page(i + kStages, s);
        }
        mma_pending = true;
        ok = mbar_wait(&sm.mma_bar, mma_phase);
        if (ok) {
            mma_phase ^= 1u;
            mma_pending = false;
        }
        tc_fence_after();

        uint32_t sv[32];
        tmem_ld_16x32bx2_x32(s_addr, sv);
        tmem_ld_wait(sv);

        int n_allow = 0;
        if ((word >> (pg & 31)) & 1u)
            n_allow = pg < own ? 64 : (pg == own ? (pos & 63) + 1 : 0);
        const int nh = min(max(n_allow - 32 * hh, 0), 32); // allowed keys in my half
        float mx = -INFINITY;
        if (crow >= 0.f) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j < nh)
                    mx = fmaxf(mx, __uint_as_float(sv[j]));
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j < nh)
                    mx = fmaxf(mx, -__uint_as_float(sv[j]));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
        if (n_allow > 0)
            mx = mx * fabsf(crow);
        float alpha = 1.f;
        bool rescale = false;
        if (n_allow > 0 && mx > m_used + kRescaleLog2) {
            if (m_used != -INFINITY) {
                alpha = ex2(m_used - mx);
                rescale = true;
                l_part *= alpha;
            }
            m_used = mx;
        }
        const float negm = n_allow > 0 ? -m_used : 0.f;
        if (__all_sync(0xFFFFFFFFu, nh == 32)) { // whole warp on full pages: no masks
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 8 * c + 2 * e;
                    const float p0 = ex2(fmaf(__uint_as_float(sv[j]), crow, negm));
                    const float p1 = ex2(fmaf(__uint_as_float(sv[j + 1]), crow, negm));
                    l_part += p0 + p1;
                    split_pair(p0, p1, hi[e], lo[e]);
                }
                const uint32_t o = swz(my_row, 4 * hh + c);
                *reinterpret_cast<uint4 *>(sm.p_hi + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(sm.p_lo + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        } else if (__all_sync(0xFFFFFFFFu, nh == 0)) { // whole warp masked out: P = 0
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t o = swz(my_row, 4 * hh + c);
                *reinterpret_cast<uint4 *>(sm.p_hi + o) = z;
                *reinterpret_cast<uint4 *>(sm.p_lo + o) = z;
            }
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 8 * c + 2 * e;
                    const float p0 = j < nh ? ex2(fmaf(__uint_as_float(sv[j]), crow, negm)) : 0.f;
                    const float p1 = j + 1 < nh ? ex2(fmaf(__uint_as_float(sv[j + 1]), crow, negm)) : 0.f;
                    l_part += p0 + p1;
                    split_pair(p0, p1, hi[e], lo[e]);
                }
                const uint32_t o = swz(my_row, 4 * hh + c);
                *reinterpret_cast<uint4 *>(sm.p_hi + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(sm.p_lo + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
        if (rescale) {
            if (hh == 0)
                sm.alpha[my_row] = alpha;
            sm.rescale = 1;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        if (sm.rescale != 0) {
            // O^T[d, r] *= alpha[r]: thread = TMEM lane = head dim d (warps of row block 0)
            if (rb == 0) {
                tc_fence_after();
                const uint32_t o_addr = tmem + (static_cast<uint32_t>(32 * qd) << 16) + kColO;
                for (int c0 = 0; c0 < Npad; c0 += 16) {
                    uint32_t o[16];
                    tmem_ld16(o_addr + c0, o);
                    tmem_ld_wait16(o);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        o[j] = __float_as_uint(__uint_as_float(o[j]) * sm.alpha[c0 + j]);
                    tmem_st16(o_addr + c0, o);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            __syncthreads(); // every thread has read sm.rescale and alpha by now
            if (rescale && hh == 0)
                sm.alpha[my_row] = 1.f;
            if (tid == 0)
                sm.rescale = 0;
        }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = sdesc_sw128(smem_u32(sm.v) + kk * 2048, 8192, 1024);
                mma_f16_ss(tmem + kColO, ad, sdesc_sw128(smem_u32(sm.p_hi) + kk * 32, 16, 1024),
                           kIdescPV, (i > 0 || kk > 0) ? 1u : 0u);
                mma_f16_ss(tmem + kColO, ad, sdesc_sw128(smem_u32(sm.p_lo) + kk * 32, 16, 1024),
                           kIdescPV, 1u);
            }
            mma_commit(&sm.mma_bar);
        }
        mma_pending = true;
    }

    bool ok = true;
    if (!aborted && mma_pending) {
        ok = mbar_wait(&sm.mma_bar, mma_phase);
        if (ok) {
            mma_phase ^= 1u;
            mma_pending = false;
        }
    }
    // row sums: combine the two halves, publish 1 / l per row
    const float l_row = l_part + __shfl_xor_sync(0xFFFFFFFFu, l_part, 16);
    if (hh == 0)
        sm.inv_l[my_row] = (row_valid && nU > 0 && l_row > 0.f) ? L.v_scale / l_row : 0.f;
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
        // O^T (lane d, column r) -> out[r][d] bf16 staged in the (free) k/v tiles, then
        // written row by row with 16-byte stores.
        uint16_t *out = reinterpret_cast<uint16_t *>(&sm.k[0][0]);
        if (rb == 0) {
            tc_fence_after();
            const int d = 32 * qd + lane;
            const uint32_t o_addr = tmem + (static_cast<uint32_t>(32 * qd) << 16) + kColO;
            for (int c0 = 0; c0 < Npad; c0 += 16) {
                uint32_t o[16];
                tmem_ld16(o_addr + c0, o);
                tmem_ld_wait16(o);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = c0 + j;
                    if (r < R) {
                        const float val = nU > 0 ? __uint_as_float(o[j]) * sm.inv_l[r] : 0.f;
                        out[r * kHeadDim + d] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
                    }
                }
            }
        }
        __syncthreads();
        for (int qn = tid; qn < R * 16; qn += NT) {
            const int r = qn >> 4, c = qn & 15;
            uint16_t *dst = L.O + (static_cast<size_t>(sm.row_tok[r]) * L.Hq + sm.row_hq[r]) * kHeadDim;
            reinterpret_cast<uint4 *>(dst)[c] = reinterpret_cast<const uint4 *>(out + r * kHeadDim)[c];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int RB>
cudaError_t launch_rb(const AttnLaunch &L, cudaStream_t st)
{
    const size_t smem = sizeof(AttnSmem<RB>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_union_attn<RB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    k_union_attn<RB><<<static_cast<unsigned>(L.n_groups), 128 * RB, smem, st>>>(L);
    return cudaGetLastError();
}

} // namespace

cudaError_t attn_launch(const AttnLaunch &L, cudaStream_t st)
{
    if (L.n_groups == 0)
        return cudaSuccess;
    // Tiles of up to 64 rows (every g * G <= 64) run on the persistent warp-specialised kernel
    // (pw_attn_ws.cu); larger tiles on the one-group-per-CTA kernel above.
    return L.g * L.G <= 64 ? attn_ws_launch(L, st) : launch_rb<2>(L, st);
}

} // namespace pw
