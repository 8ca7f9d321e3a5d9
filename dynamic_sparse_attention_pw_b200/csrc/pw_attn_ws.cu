// pw_attn_ws.cu -- persistent, warp-specialised ID-aware union attention (tiles of <= 64 rows).
//
// Same arithmetic as the one-group-per-CTA kernel in pw_attn.cu ("PageWeaver: KV-Guided Query
// Unions for Sparse Attention", Abstract: union pages loaded once per group, each query masked
// to its own support, complete output per query, FP8 KV), organised so that the tensor-core
// work of one page overlaps the decode and softmax work of its neighbours.
//
// One CTA per SM walks the groups blockIdx.x, blockIdx.x + gridDim.x, ... .  Its warps:
//   warps 0-7    decode   Q tile of each group (bf16, gathered by query ID); E4M3 K and V
//                         pages -> bf16 operand tiles
//   warps 8-11   softmax  S -> P for each page, lazy O^T rescale, epilogue of each group
//   warp 12      load     bulk copies (TMA) of the union pages into a 3-stage FP8 ring
//   warp 13      MMA      S_i = Q K_i^T issued one page ahead of O^T += V_{i-1}^T P_{i-1}^T
// O^T = V^T P^T puts the head dimension on the 128 MMA rows; P_hi and P_lo are stacked along N
// (N = 2 * rows), so one product per k-step reads V once and accumulates both halves, which the
// epilogue adds.  K and V have separate buffers: a K slot is free once S is done, a V slot
// once the product is done.  Every hand-off is an mbarrier; every wait is bounded and, when it
// runs out, sets an abort flag that releases the other roles.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pw_attn_common.cuh"
#include "pw_internal.h"
#include "pw_sm100.cuh"

namespace pw {
namespace {

using namespace attn;

constexpr int kNS = 3;        // FP8 page stages
constexpr int kNK = 2;        // bf16 K slots
constexpr int kNV = 3;        // bf16 V slots
constexpr int kDecThreads = 256;
constexpr int kWarpSm0 = 8, kWarpLoad = 12, kWarpMma = 13;
constexpr int kThreads = 448; // 14 warps
constexpr uint32_t kTmemCols = 512; // S[0..1] at columns 0 / 64, O^T[0..1] at 128 / 256
constexpr uint32_t kColO = 128;
constexpr uint32_t kIdescS = idesc_bf16_f32(64, 64, false, false);
constexpr uint32_t kFull = 0xFFFFFFFFu;

struct __align__(1024) WsSmem {
    uint8_t q[2][2][64 * 128];   // [Q buffer][dim-block][64 rows][128 B]
    uint8_t k[kNK][2][64 * 128]; // [slot][dim-block][64 keys][128 B]
    uint8_t v[kNV][2][64 * 128];
    uint8_t p[2][128 * 128];     // [buffer][P_hi rows 0..npad-1, P_lo rows npad..2npad-1][64 keys]
    uint8_t stage_k[kNS][kPageBytes];
    uint8_t stage_v[kNS][kPageBytes];
    uint16_t out[64 * 128];      // epilogue staging, bf16 [row][head dim]
    float alpha[2][64];
    float inv_l[64];
    int32_t row_tok[64];
    int32_t row_hq[64];
    uint64_t full_stage[kNS], empty_stage[kNS];
    uint64_t k_full[kNK], k_empty[kNK];
    uint64_t v_full[kNV], v_empty[kNV];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2];
    uint64_t o_bar;
    uint64_t q_full[2], q_empty[2];
    uint64_t o_free[2];
    uint64_t drain_bar;
    uint32_t load_issued; // pages whose copies the load warp issued (for the abort drain)
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t early_exit;
};

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int32_t *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*reinterpret_cast<volatile int32_t *>(abort_flag) != 0)
            return false;
        if (clock64() - t0 > kWaitCycles) {
            *reinterpret_cast<volatile int32_t *>(abort_flag) = 1;
            return false;
        }
    }
    return true;
}

// Named barrier 1 over the 128 softmax threads, returning whether any of them passed `pred`.
__device__ __forceinline__ bool softmax_bar_or(bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 q, %1, 0;\n\t"
                 "bar.red.or.pred p, 1, 128, q;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}\n"
                 : "=r"(r)
                 : "r"(pred ? 1u : 0u)
                 : "memory");
    return r != 0;
}

__device__ __forceinline__ void softmax_bar()
{
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// A descriptor's start-address field is (address >> 4) in its low 14 bits: a descriptor for
// `base + off` is the descriptor for `base` plus off >> 4 (no carry below 256 KiB).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t off_bytes)
{
    return d + static_cast<uint64_t>(off_bytes >> 4);
}

struct PendingPV {
    uint32_t it, vs, ob, nact, npad;
    bool first;
};

__global__ void __launch_bounds__(kThreads, 1) k_union_attn_ws(const AttnLaunch L)
{
    extern __shared__ uint8_t smem_raw[];
    WsSmem &sm = *reinterpret_cast<WsSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0)
        sm.early_exit = *reinterpret_cast<volatile int32_t *>(L.status) == PW_ERR_TIMEOUT ? 1 : 0;
    __syncthreads();
    if (sm.early_exit != 0)
        return;

    if (tid == 0) {
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&sm.full_stage[s], 1);
            mbar_init(&sm.empty_stage[s], kDecThreads);
        }
        for (int s = 0; s < kNK; ++s) {
            mbar_init(&sm.k_full[s], kDecThreads);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int s = 0; s < kNV; ++s) {
            mbar_init(&sm.v_full[s], kDecThreads);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.s_full[s], 1);
            mbar_init(&sm.s_empty[s], 128);
            mbar_init(&sm.p_full[s], 128);
            mbar_init(&sm.q_full[s], kDecThreads);
            mbar_init(&sm.q_empty[s], 1);
            mbar_init(&sm.o_free[s], 128);
        }
        mbar_init(&sm.o_bar, 1);
        mbar_init(&sm.drain_bar, 1);
        sm.abort_flag = 0;
        sm.load_issued = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int64_t g0 = blockIdx.x, gstep = gridDim.x;

    if (warp == kWarpLoad) {
        // ---------------- load: union pages -> FP8 stages ----------------
        uint32_t it = 0;
        bool stop = false;
        for (int64_t gi = g0; gi < L.n_groups && !stop; gi += gstep) {
            const int b = L.gmeta[3 * gi], h = L.gmeta[3 * gi + 1];
            const int u0 = L.union_off[gi], nU = L.union_off[gi + 1] - u0;
            for (int j0 = 0; j0 < nU && !stop; j0 += 32) {
                int phys = 0;
                if (j0 + lane < nU) {
                    const int pg = L.union_pages[u0 + j0 + lane];
                    phys = L.page_table[static_cast<size_t>(b) * L.max_pages + pg];
                    if (phys < 0 || phys >= L.n_phys) {
                        set_status(L.status, PW_ERR_INVALID_ARG);
                        phys = 0;
                    }
                }
                const int cnt = min(32, nU - j0);
                for (int jj = 0; jj < cnt; ++jj, ++it) {
                    const int ph = __shfl_sync(kFull, phys, jj);
                    int ok = 1;
                    if (lane == 0) {
                        const uint32_t st = it % kNS;
                        ok = wait_bar(&sm.empty_stage[st], ((it / kNS) & 1u) ^ 1u, &sm.abort_flag);
                        if (ok) {
                            const size_t off = (static_cast<size_t>(ph) * L.Hkv + h) * kPageBytes;
                            mbar_arrive_expect_tx(&sm.full_stage[st], 2 * kPageBytes);
                            bulk_g2s(sm.stage_k[st], L.K + off, kPageBytes, &sm.full_stage[st]);
                            bulk_g2s(sm.stage_v[st], L.V + off, kPageBytes, &sm.full_stage[st]);
                            sm.load_issued = it + 1;
                        }
                    }
                    if (__shfl_sync(kFull, ok, 0) == 0) {
                        stop = true;
                        break;
                    }
                }
            }
        }
    } else if (warp == kWarpMma) {
        // ---------------- MMA issue: the warp runs in lockstep, one elected lane issues ----------------
        // Lane 0 does the waits and broadcasts the outcome, so every decision is warp-uniform;
        // operands are computed by the converged warp (uniform registers), the elected lane
        // (always lane 0) issues the MMAs and their commits.
        auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            int ok = 1;
            if (lane == 0)
                ok = wait_bar(bar, parity, &sm.abort_flag);
            return __shfl_sync(kFull, ok, 0) != 0;
        };
        const uint64_t dsw = sdesc_sw128(0u, 16, 1024);    // K-major, address added below
        const uint64_t dmn = sdesc_sw128(0u, 8192, 1024);  // MN-major V^T
        uint32_t it = 0, nact = 0;
        bool have_prev = false, ok = true;
        PendingPV prev{};
        auto issue_pv = [&](const PendingPV &p) -> bool {
            const uint32_t pb = p.it & 1u;
            if (!wwait(&sm.p_full[pb], (p.it >> 1) & 1u) || !wwait(&sm.v_full[p.vs], (p.it / kNV) & 1u))
                return false;
            if (p.first && !wwait(&sm.o_free[p.ob], ((p.nact >> 1) & 1u) ^ 1u))
                return false;
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, static_cast<int>(2 * p.npad), true, false);
            const uint32_t d = tmem + kColO + 128 * p.ob;
            const uint64_t ad = desc_add(dmn, smem_u32(&sm.v[p.vs][0][0]));
            const uint64_t bd = desc_add(dsw, smem_u32(sm.p[pb]));
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16_ss(d, ad + 128u * kk, bd + 2u * kk, idesc, (p.first && kk == 0) ? 0u : 1u);
                mma_commit(&sm.v_empty[p.vs]);
                mma_commit(&sm.o_bar);
            }
            __syncwarp();
            return true;
        };
        for (int64_t gi = g0; gi < L.n_groups && ok; gi += gstep) {
            const int R = L.gsize[gi] * L.G;
            const uint32_t npad = static_cast<uint32_t>((R + 15) & ~15);
            const int u0 = L.union_off[gi], nU = L.union_off[gi + 1] - u0;
            if (nU == 0)
                continue;
            const uint32_t qb = nact & 1u;
            if (!wwait(&sm.q_full[qb], (nact >> 1) & 1u)) {
                ok = false;
                break;
            }
            const uint64_t aq0 = desc_add(dsw, smem_u32(sm.q[qb][0]));
            const uint64_t aq1 = desc_add(dsw, smem_u32(sm.q[qb][1]));
            for (int j = 0; j < nU; ++j, ++it) {
                const uint32_t ks = it % kNK, sb = it & 1u;
                if (!wwait(&sm.k_full[ks], (it / kNK) & 1u) ||
                    !wwait(&sm.s_empty[sb], ((it >> 1) & 1u) ^ 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t bk0 = desc_add(dsw, smem_u32(sm.k[ks][0]));
                const uint64_t bk1 = desc_add(dsw, smem_u32(sm.k[ks][1]));
                const uint32_t ds = tmem + 64 * sb;
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ss(ds, aq0 + 2u * kk, bk0 + 2u * kk, kIdescS, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ss(ds, aq1 + 2u * kk, bk1 + 2u * kk, kIdescS, 1u);
                    mma_commit(&sm.s_full[sb]);
                    mma_commit(&sm.k_empty[ks]);
                    if (j == nU - 1)
                        mma_commit(&sm.q_empty[qb]);
                }
                __syncwarp();
                if (have_prev && !issue_pv(prev)) {
                    ok = false;
                    break;
                }
                prev = PendingPV{it, it % kNV, nact & 1u, nact, npad, j == 0};
                have_prev = true;
            }
            ++nact;
        }
        if (ok && have_prev)
            (void)issue_pv(prev);
    } else if (warp < kWarpSm0) {
        // ---------------- decode: Q tiles and E4M3 -> bf16 K/V tiles (256 threads) ----------------
        uint32_t it = 0, nact = 0;
        bool ok = true;
        for (int64_t gi = g0; gi < L.n_groups && ok; gi += gstep) {
            const int h = L.gmeta[3 * gi + 1];
            const int R = L.gsize[gi] * L.G;
            const int u0 = L.union_off[gi], nU = L.union_off[gi + 1] - u0;
            if (nU == 0)
                continue;
            const uint32_t qb = nact & 1u;
            if (!wait_bar(&sm.q_empty[qb], ((nact >> 1) & 1u) ^ 1u, &sm.abort_flag)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int rep = 0; rep < 4; ++rep) {
                const int qn = tid + kDecThreads * rep;
                const int row = qn >> 4, c = qn & 15;
                uint4 val = make_uint4(0u, 0u, 0u, 0u);
                if (row < R) {
                    const int mi = row / L.G;
                    const int64_t tok = L.qids[gi * L.g + mi];
                    const int hq = h * L.G + (row - mi * L.G);
                    val = __ldg(reinterpret_cast<const uint4 *>(
                                    L.Q + (static_cast<size_t>(tok) * L.Hq + hq) * kHeadDim) + c);
                }
                *reinterpret_cast<uint4 *>(sm.q[qb][c >> 3] + swz(row, c & 7)) = val;
            }
            fence_proxy_async_smem();
            mbar_arrive(&sm.q_full[qb]);
            for (int j = 0; j < nU; ++j, ++it) {
                const uint32_t st = it % kNS, ks = it % kNK, vs = it % kNV;
                if (!wait_bar(&sm.full_stage[st], (it / kNS) & 1u, &sm.abort_flag) ||
                    !wait_bar(&sm.k_empty[ks], ((it / kNK) & 1u) ^ 1u, &sm.abort_flag)) {
                    ok = false;
                    break;
                }
                decode_page<kDecThreads>(sm.stage_k[st], sm.k[ks], tid);
                fence_proxy_async_smem();
                mbar_arrive(&sm.k_full[ks]);
                if (!wait_bar(&sm.v_empty[vs], ((it / kNV) & 1u) ^ 1u, &sm.abort_flag)) {
                    ok = false;
                    break;
                }
                decode_page<kDecThreads>(sm.stage_v[st], sm.v[vs], tid);
                fence_proxy_async_smem();
                mbar_arrive(&sm.v_full[vs]);
                mbar_arrive(&sm.empty_stage[st]);
            }
            ++nact;
        }
    } else {
        // ---------------- softmax + epilogue (128 threads, warps 8-11) ----------------
        const int st = tid - kWarpSm0 * 32; // 0..127, also the TMEM lane (head dim) in the epilogue
        const int qd = warp - kWarpSm0;     // TMEM lane quadrant
        const int row = 16 * qd + (lane & 15);
        const int hh = lane >> 4;
        const float crow = L.sm_scale * L.k_scale * kLog2e;
        const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
        uint32_t it = 0, nact = 0;
        // Products (one o_bar phase per page) known complete: [0, pv_done).  A parity wait is
        // only unambiguous one phase ahead of what is known complete, so wait_pv steps through
        // the phases in order.  Seeing S of page i also proves the product of page i-2 complete
        // (S_i is issued after it).
        uint32_t pv_done = 0;
        auto wait_pv = [&](uint32_t x) -> bool { // product of page x complete
            for (; pv_done <= x; ++pv_done)
                if (!wait_bar(&sm.o_bar, pv_done & 1u, &sm.abort_flag))
                    return false;
            return true;
        };
        bool ok = true;
        for (int64_t gi = g0; gi < L.n_groups && ok; gi += gstep) {
            const int b = L.gmeta[3 * gi], h = L.gmeta[3 * gi + 1];
            const int R = L.gsize[gi] * L.G;
            const int npad = (R + 15) & ~15;
            const int u0 = L.union_off[gi], nU = L.union_off[gi + 1] - u0;
            const bool valid = row < R;
            int64_t tok = 0;
            int hq = 0, pos = 0, own = 0;
            const uint32_t *bitrow = nullptr;
            if (valid) {
                const int mi = row / L.G;
                tok = L.qids[gi * L.g + mi];
                hq = h * L.G + (row - mi * L.G);
                pos = static_cast<int>(tok - L.cu[b]);
                own = pos >> 6;
                bitrow = L.bits + (static_cast<size_t>(tok) * L.Hkv + h) * L.words;
            }
            if (hh == 0) {
                sm.row_tok[row] = static_cast<int32_t>(tok);
                sm.row_hq[row] = hq;
            }
            if (nU == 0) {
                if (valid) { // no union page: every row of the group is empty
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        L.O + (static_cast<size_t>(tok) * L.Hq + hq) * kHeadDim + 64 * hh);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        dst[c] = make_uint4(0u, 0u, 0u, 0u);
                }
                softmax_bar();
                continue;
            }
            const uint32_t ob = nact & 1u;
            const uint32_t o_addr = tmem + lane_base + kColO + 128 * ob;
            float m_used = -INFINITY, l_part = 0.f;
            int pg_next = L.union_pages[u0];
            uint32_t word_next = valid ? __ldg(bitrow + (pg_next >> 5)) : 0u;
            for (int j = 0; j < nU; ++j, ++it) {
                const int pg = pg_next;
                const uint32_t word = word_next;
                if (j + 1 < nU) { // next page's id and my membership word, fetched early
                    pg_next = L.union_pages[u0 + j + 1];
                    word_next = valid ? __ldg(bitrow + (pg_next >> 5)) : 0u;
                }
                const uint32_t sb = it & 1u, pb = it & 1u;
                // every abort decision of this role is collective: a thread that left alone
                // would strand the others at the named barrier or in a warp-wide TMEM load
                ok = wait_bar(&sm.s_full[sb], (it >> 1) & 1u, &sm.abort_flag);
                if (softmax_bar_or(!ok)) {
                    ok = false;
                    break;
                }
                if (it >= 2 && pv_done < it - 1)
                    pv_done = it - 1;
                tc_fence_after();
                uint32_t sv[32];
                tmem_ld_16x32bx2_x32(tmem + lane_base + 64 * sb, sv);
                tmem_ld_wait(sv);
                tc_fence_before();
                mbar_arrive(&sm.s_empty[sb]);

                int n_allow = 0;
                if ((word >> (pg & 31)) & 1u)
                    n_allow = pg < own ? 64 : (pg == own ? (pos & 63) + 1 : 0);
                const int nh = min(max(n_allow - 32 * hh, 0), 32);
                float mx = -INFINITY;
                if (crow >= 0.f) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e < nh)
                            mx = fmaxf(mx, __uint_as_float(sv[e]));
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e < nh)
                            mx = fmaxf(mx, -__uint_as_float(sv[e]));
                }
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
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
                // P buffer pb was last read by the product of page it-2, complete since
                // S of page it (issued after it) is.
                // Rows 0..npad-1 hold P_hi, rows npad..2 npad-1 P_lo; only rows < npad write.
                uint8_t *phi = sm.p[pb], *plo = sm.p[pb] + npad * 128;
                if (__all_sync(kFull, nh == 32)) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int x = 8 * c + 2 * e;
                            const float p0 = ex2(fmaf(__uint_as_float(sv[x]), crow, negm));
                            const float p1 = ex2(fmaf(__uint_as_float(sv[x + 1]), crow, negm));
                            l_part += p0 + p1;
                            split_pair(p0, p1, hi[e], lo[e]);
                        }
                        const uint32_t o = swz(row, 4 * hh + c);
                        if (row < npad) {
                            *reinterpret_cast<uint4 *>(phi + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                            *reinterpret_cast<uint4 *>(plo + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        }
                    }
                } else if (__all_sync(kFull, nh == 0)) {
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t o = swz(row, 4 * hh + c);
                        if (row < npad) {
                            *reinterpret_cast<uint4 *>(phi + o) = z;
                            *reinterpret_cast<uint4 *>(plo + o) = z;
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int x = 8 * c + 2 * e;
                            const float p0 = x < nh ? ex2(fmaf(__uint_as_float(sv[x]), crow, negm)) : 0.f;
                            const float p1 = x + 1 < nh ? ex2(fmaf(__uint_as_float(sv[x + 1]), crow, negm)) : 0.f;
                            l_part += p0 + p1;
                            split_pair(p0, p1, hi[e], lo[e]);
                        }
                        const uint32_t o = swz(row, 4 * hh + c);
                        if (row < npad) {
                            *reinterpret_cast<uint4 *>(phi + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                            *reinterpret_cast<uint4 *>(plo + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        }
                    }
                }
                if (hh == 0)
                    sm.alpha[pb][row] = rescale ? alpha : 1.f;
                fence_proxy_async_smem();
                if (softmax_bar_or(rescale)) {
                    // O^T[d, r] *= alpha[r] for both accumulator halves, after the previous
                    // page's product (the only one that may still run: S of this page, issued
                    // after the products before it, is complete).
                    ok = j == 0 || wait_pv(it - 1);
                    if (softmax_bar_or(!ok)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int c0 = 0; c0 < 2 * npad; c0 += 16) {
                        uint32_t o[16];
                        tmem_ld16(o_addr + c0, o);
                        tmem_ld_wait16(o);
                        const int r0 = c0 < npad ? c0 : c0 - npad;
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * sm.alpha[pb][r0 + e]);
                        tmem_st16(o_addr + c0, o);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(&sm.p_full[pb]);
            }
            if (!ok)
                break;
            // epilogue: the group's last product is page it - 1
            ok = wait_pv(it - 1);
            const float l_row = l_part + __shfl_xor_sync(kFull, l_part, 16);
            if (hh == 0)
                sm.inv_l[row] = (valid && l_row > 0.f) ? L.v_scale / l_row : 0.f;
            if (softmax_bar_or(!ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int c0 = 0; c0 < npad; c0 += 16) {
                uint32_t ohi[16], olo[16];
                tmem_ld16(o_addr + c0, ohi);
                tmem_ld16(o_addr + npad + c0, olo);
                tmem_ld_wait16(ohi);
                tmem_ld_wait16(olo);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int r = c0 + e;
                    const float val = (__uint_as_float(ohi[e]) + __uint_as_float(olo[e])) * sm.inv_l[r];
                    sm.out[r * kHeadDim + st] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.o_free[ob]);
            softmax_bar();
            for (int qn = st; qn < R * 16; qn += 128) {
                const int r = qn >> 4, c = qn & 15;
                uint16_t *dst = L.O + (static_cast<size_t>(sm.row_tok[r]) * L.Hq + sm.row_hq[r]) * kHeadDim;
                reinterpret_cast<uint4 *>(dst)[c] =
                    reinterpret_cast<const uint4 *>(sm.out + r * kHeadDim)[c];
            }
            softmax_bar(); // row_tok, inv_l and out are rewritten by the next group
            ++nact;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (sm.abort_flag != 0) {
        set_status(L.status, PW_ERR_TIMEOUT);
        // Let copies and products still in flight land before the CTA exits (bounded waits):
        // the last copy issued on each stage, and every product issued so far.
        if (tid == 0) {
            const uint32_t n = sm.load_issued;
            for (uint32_t s = 0; s < kNS && s < n; ++s) {
                const uint32_t last = s + ((n - 1 - s) / kNS) * kNS;
                (void)mbar_wait(&sm.full_stage[s], (last / kNS) & 1u);
            }
        }
        if (warp == kWarpMma) {
            if (elect_one()) {
                mma_commit(&sm.drain_bar);
                (void)mbar_wait(&sm.drain_bar, 0);
            }
            __syncwarp();
        }
    }
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

} // namespace

cudaError_t attn_ws_launch(const AttnLaunch &L, cudaStream_t st)
{
    if (L.n_groups == 0)
        return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const size_t smem = sizeof(WsSmem) + 1024;
    e = cudaFuncSetAttribute(k_union_attn_ws, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    const int64_t grid = L.n_groups < sms ? L.n_groups : sms;
    k_union_attn_ws<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(L);
    return cudaGetLastError();
}

} // namespace pw
