// pw_group.cu -- the bounded GPU search of PageWeaver ("PageWeaver: KV-Guided Query Unions for
// Sparse Attention", Abstract: a bounded GPU search produces query IDs; AI Radio episode on the
// paper, paper summary: greedy inside a bounded window, collecting queries whose selected sets
// add few new pages, with the execution size g fixed independently of W).
//
// Four launches on the caller's stream:
//   k_bitsets        sel_pages -> per-(token, kv head) page bitsets + set sizes (validation)
//   k_greedy<..>     one warp per (sequence, kv head, window): ballot/popcount greedy
//   k_union_offsets  exclusive scan of the union sizes -> CSR offsets
//   k_union_pages    union bitsets -> ascending page lists
#include <cstdint>
#include <cuda_runtime.h>

#include "pw_internal.h"
#include "pw_sm100.cuh"

namespace pw {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ int seq_of_token(const int32_t *cu, int B, int64_t t)
{
    int lo = 0, hi = B;
    while (lo < hi) { // largest b with cu[b] <= t
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------------------------------
// k_bitsets: one warp per token, all kv heads.  Invalid ids (outside [-1, own page]) are
// reported and skipped.  counts[t, h] = |S(t, h)| (distinct pages).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_bitsets(const int32_t *__restrict__ sel,
                                                 const int32_t *__restrict__ cu, int B, int64_t T,
                                                 int Hkv, int kmax, int words,
                                                 uint32_t *__restrict__ bits,
                                                 uint16_t *__restrict__ counts, int32_t *status)
{
    extern __shared__ uint32_t sh_acc[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    uint32_t *acc = sh_acc + wib * words;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + wib; t < T;
         t += nwarps) {
        const int b = seq_of_token(cu, B, t);
        const int own = static_cast<int>((t - cu[b]) >> 6);
        for (int h = 0; h < Hkv; ++h) {
            for (int w = lane; w < words; w += 32)
                acc[w] = 0;
            __syncwarp();
            const int32_t *row = sel + (static_cast<size_t>(t) * Hkv + h) * kmax;
            for (int j = lane; j < kmax; j += 32) {
                const int32_t p = row[j];
                if (p == -1)
                    continue;
                if (p < -1 || p > own) {
                    set_status(status, PW_ERR_BAD_SELECTION);
                    continue;
                }
                atomicOr(&acc[p >> 5], 1u << (p & 31));
            }
            __syncwarp();
            uint32_t cnt = 0;
            uint32_t *out = bits + (static_cast<size_t>(t) * Hkv + h) * words;
            for (int w = lane; w < words; w += 32) {
                const uint32_t v = acc[w];
                out[w] = v;
                cnt += __popc(v);
            }
            cnt = __reduce_add_sync(kFull, cnt);
            if (lane == 0)
                counts[static_cast<size_t>(t) * Hkv + h] = static_cast<uint16_t>(cnt);
            __syncwarp();
        }
    }
}

// ---------------------------------------------------------------------------------------
// Window enumeration: windows are ordered (b, h, w); groups likewise, W / g per full window
// and ceil(n / g) for a final partial window of n tokens.
// ---------------------------------------------------------------------------------------
struct Window {
    int b, h, w, n, nwb;
    int64_t tok0, gbase;
};

__device__ __forceinline__ Window locate_window(int64_t widx, const int32_t *cu, int B, int Hkv,
                                                int W, int g)
{
    Window r{0, 0, 0, 0, 0, 0, 0};
    int64_t gacc = 0;
    for (int b = 0; b < B; ++b) {
        const int len = cu[b + 1] - cu[b];
        const int nwin = (len + W - 1) / W;
        const int64_t gpb = static_cast<int64_t>(len / W) * (W / g) + ((len % W) + g - 1) / g;
        const int64_t wpb = static_cast<int64_t>(nwin) * Hkv;
        if (widx < wpb) {
            r.b = b;
            r.h = static_cast<int>(widx / nwin);
            r.w = static_cast<int>(widx % nwin);
            r.tok0 = cu[b] + static_cast<int64_t>(r.w) * W;
            r.n = min(W, len - r.w * W);
            r.nwb = (((len + 63) >> 6) + 31) >> 5;
            r.gbase = gacc + r.h * gpb + static_cast<int64_t>(r.w) * (W / g);
            return r;
        }
        widx -= wpb;
        gacc += gpb * Hkv;
    }
    return r;
}

// cost[k] -= |S(c_k) & X| for the warp's available candidates, X given word-distributed
// (lane l holds word l + 32 j in x[j]); only the non-zero words of X are visited.
template <int KPL, int WPL>
__device__ __forceinline__ void subtract_overlap(const uint32_t (&x)[WPL], const uint32_t *sb,
                                                 int stride, int lane, uint32_t avail,
                                                 int (&cost)[KPL])
{
#pragma unroll
    for (int j = 0; j < WPL; ++j) {
        uint32_t nz = __ballot_sync(kFull, x[j] != 0u);
        while (nz) {
            const int src = __ffs(nz) - 1;
            nz &= nz - 1;
            const uint32_t xw = __shfl_sync(kFull, x[j], src);
            const uint32_t *row = sb + (src + 32 * j) * stride;
#pragma unroll
            for (int k = 0; k < KPL; ++k)
                if ((avail >> k) & 1u)
                    cost[k] -= __popc(row[lane + 32 * k] & xw);
        }
    }
}

// ---------------------------------------------------------------------------------------
// k_greedy: one warp per window.  The window's bitsets sit in shared memory transposed
// ([word][candidate], stride W + 1), so lanes that own consecutive candidates read
// consecutive words.  Lane l owns candidates l, l + 32, ... (KPL of them) and union words
// l, l + 32, ... (WPL of them).  Costs are maintained incrementally:
//   at a seed:  cost(c) = |S(c)| - |S(c) & S(seed)|
//   at a pick:  cost(c) -= |S(c) & (S(pick) \ U)|   and U |= S(pick)
// which equals |S(c) \ U| at every step.  argmin(cost, index) is one redux.sync.min over the
// packed key (cost << 16 | index), so ties go to the lowest token index.
// ---------------------------------------------------------------------------------------
template <int KPL, int WPL>
__global__ void __launch_bounds__(128) k_greedy(
    const uint32_t *__restrict__ bits, const uint16_t *__restrict__ counts,
    const int32_t *__restrict__ cu, int B, int Hkv, int words, int W, int g,
    int64_t n_windows, int32_t *__restrict__ qids, int32_t *__restrict__ gsize,
    int32_t *__restrict__ gmeta, uint32_t *__restrict__ ubits, int32_t *__restrict__ ucount)
{
    extern __shared__ uint32_t sh_win[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int stride = W + 1;
    uint32_t *sb = sh_win + static_cast<size_t>(wib) * words * stride;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);

    for (int64_t widx = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + wib;
         widx < n_windows; widx += nwarps) {
        const Window win = locate_window(widx, cu, B, Hkv, W, g);
        const int n = win.n, nwb = win.nwb;
        // stage the window's bitsets, transposed
        const int total = n * nwb;
        for (int q = lane; q < total; q += 32) {
            const int c = q / nwb, w = q - c * nwb;
            sb[w * stride + c] =
                bits[(static_cast<size_t>(win.tok0 + c) * Hkv + win.h) * words + w];
        }
        int cnt[KPL];
        uint32_t avail = 0;
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int c = lane + 32 * k;
            cnt[k] = 0;
            if (c < n) {
                avail |= 1u << k;
                cnt[k] = counts[static_cast<size_t>(win.tok0 + c) * Hkv + win.h];
            }
        }
        __syncwarp();

        int remaining = n;
        int64_t gidx = win.gbase;
        while (remaining > 0) {
            // seed: lowest unassigned token of the window
            uint32_t mine = 0xFFFFFFFFu;
#pragma unroll
            for (int k = KPL - 1; k >= 0; --k)
                if ((avail >> k) & 1u)
                    mine = lane + 32 * k;
            const uint32_t seed = __reduce_min_sync(kFull, mine);
            uint32_t memb = 0;
            if (static_cast<int>(seed & 31u) == lane) {
                avail &= ~(1u << (seed >> 5));
                memb |= 1u << (seed >> 5);
            }
            --remaining;
            int m = 1;
            uint32_t U[WPL];
#pragma unroll
            for (int j = 0; j < WPL; ++j) {
                const int w = lane + 32 * j;
                U[j] = w < nwb ? sb[w * stride + seed] : 0u;
            }
            int cost[KPL];
#pragma unroll
            for (int k = 0; k < KPL; ++k)
                cost[k] = cnt[k];
            subtract_overlap<KPL, WPL>(U, sb, stride, lane, avail, cost);

            while (m < g && remaining > 0) {
                uint32_t key = 0xFFFFFFFFu;
#pragma unroll
                for (int k = 0; k < KPL; ++k)
                    if ((avail >> k) & 1u)
                        key = min(key, (static_cast<uint32_t>(cost[k]) << 16) |
                                           static_cast<uint32_t>(lane + 32 * k));
                key = __reduce_min_sync(kFull, key);
                const uint32_t c = key & 0xFFFFu;
                if (static_cast<int>(c & 31u) == lane) {
                    avail &= ~(1u << (c >> 5));
                    memb |= 1u << (c >> 5);
                }
                --remaining;
                ++m;
                uint32_t Dlt[WPL];
#pragma unroll
                for (int j = 0; j < WPL; ++j) {
                    const int w = lane + 32 * j;
                    const uint32_t s = w < nwb ? sb[w * stride + c] : 0u;
                    Dlt[j] = s & ~U[j];
                    U[j] |= s;
                }
                subtract_overlap<KPL, WPL>(Dlt, sb, stride, lane, avail, cost);
            }

            // emit: members ascending (candidate index = lane + 32 k, so k-major then lane)
            int out = 0;
            int32_t *q = qids + gidx * g;
#pragma unroll
            for (int k = 0; k < KPL; ++k) {
                const uint32_t bal = __ballot_sync(kFull, (memb >> k) & 1u);
                if ((memb >> k) & 1u) {
                    const int slot = out + __popc(bal & ((1u << lane) - 1u));
                    q[slot] = static_cast<int32_t>(win.tok0 + lane + 32 * k);
                }
                out += __popc(bal);
            }
            for (int i = m + lane; i < g; i += 32)
                q[i] = -1;
            uint32_t pc = 0;
#pragma unroll
            for (int j = 0; j < WPL; ++j) {
                const int w = lane + 32 * j;
                if (w < words)
                    ubits[gidx * words + w] = U[j];
                pc += __popc(U[j]);
            }
            pc = __reduce_add_sync(kFull, pc);
            if (lane == 0) {
                gsize[gidx] = m;
                gmeta[3 * gidx + 0] = win.b;
                gmeta[3 * gidx + 1] = win.h;
                gmeta[3 * gidx + 2] = win.w;
                ucount[gidx] = static_cast<int32_t>(pc);
            }
            ++gidx;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------------------
// k_union_offsets: single block; exclusive scan of ucount -> union_off[0..n].  Thread t owns
// the contiguous range [t c, (t + 1) c), c a multiple of 4, read and written as int4 where both
// arrays are 16-byte aligned: one pass for the range sums, a block scan of the sums, one pass
// for the offsets.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_union_offsets(const int32_t *__restrict__ ucount,
                                                        int64_t n, int64_t cap,
                                                        int32_t *__restrict__ union_off,
                                                        int32_t *status)
{
    __shared__ long long wsum[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t chunk = ((n + blockDim.x - 1) / blockDim.x + 3) & ~static_cast<int64_t>(3);
    const int64_t s = min(n, static_cast<int64_t>(tid) * chunk);
    const int64_t e = min(n, s + chunk);
    const bool vec = ((reinterpret_cast<uintptr_t>(ucount) | reinterpret_cast<uintptr_t>(union_off)) & 15) == 0;
    const int64_t ev = vec ? s + ((e - s) & ~static_cast<int64_t>(3)) : s; // end of the int4 part
    long long local = 0;
    for (int64_t i = s; i < ev; i += 4) {
        const int4 v = *reinterpret_cast<const int4 *>(ucount + i);
        local += static_cast<long long>(v.x) + v.y + v.z + v.w;
    }
    for (int64_t i = ev; i < e; ++i)
        local += ucount[i];
    long long incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long v = __shfl_up_sync(kFull, incl, off);
        if (lane >= off)
            incl += v;
    }
    if (lane == 31)
        wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        long long v = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long u = __shfl_up_sync(kFull, v, off);
            if (lane >= off)
                v += u;
        }
        if (lane < nw)
            wsum[lane] = v;
    }
    __syncthreads();
    long long base = (warp > 0 ? wsum[warp - 1] : 0) + incl - local;
    for (int64_t i = s; i < ev; i += 4) {
        const int4 v = *reinterpret_cast<const int4 *>(ucount + i);
        int4 o;
        o.x = static_cast<int32_t>(base);
        o.y = static_cast<int32_t>(base + v.x);
        o.z = static_cast<int32_t>(base + v.x + v.y);
        o.w = static_cast<int32_t>(base + v.x + v.y + v.z);
        base += static_cast<long long>(v.x) + v.y + v.z + v.w;
        *reinterpret_cast<int4 *>(union_off + i) = o;
    }
    for (int64_t i = ev; i < e; ++i) {
        union_off[i] = static_cast<int32_t>(base);
        base += ucount[i];
    }
    if (tid == 0) {
        const long long total = wsum[(blockDim.x >> 5) - 1];
        union_off[n] = static_cast<int32_t>(total);
        if (total > cap)
            set_status(status, PW_ERR_CAPACITY);
    }
}

// ---------------------------------------------------------------------------------------
// k_union_pages: one warp per group; bitset words -> ascending page ids.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_union_pages(const uint32_t *__restrict__ ubits,
                                                     const int32_t *__restrict__ union_off,
                                                     int64_t n, int words, int64_t cap,
                                                     int32_t *__restrict__ union_pages)
{
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t gi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         gi < n; gi += nwarps) {
        int64_t o = union_off[gi];
        for (int w0 = 0; w0 < words; w0 += 32) {
            const int w = w0 + lane;
            uint32_t v = w < words ? ubits[gi * words + w] : 0u;
            const int c = __popc(v);
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int u = __shfl_up_sync(kFull, incl, off);
                if (lane >= off)
                    incl += u;
            }
            int64_t dst = o + incl - c;
            while (v) {
                const int bit = __ffs(v) - 1;
                v &= v - 1;
                if (dst < cap)
                    union_pages[dst] = w * 32 + bit;
                ++dst;
            }
            o += __shfl_sync(kFull, incl, 31);
        }
    }
}

template <int KPL, int WPL>
cudaError_t launch_greedy(const GroupLaunch &L, cudaStream_t st, int warps, size_t smem)
{
    auto kern = k_greedy<KPL, WPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    const int64_t blocks64 = (L.n_windows + warps - 1) / warps;
    const int blocks = static_cast<int>(blocks64 < 1048576 ? blocks64 : 1048576);
    kern<<<blocks, warps * 32, smem, st>>>(L.bits, L.counts, L.cu, L.B, L.Hkv, L.words, L.W, L.g,
                                           L.n_windows, L.qids, L.gsize, L.gmeta, L.ubits,
                                           L.ucount);
    return cudaGetLastError();
}

} // namespace

cudaError_t group_launch(const GroupLaunch &L, cudaStream_t st)
{
    cudaError_t e;
    // 1. bitsets
    {
        const int warps = 8;
        const size_t smem = static_cast<size_t>(warps) * L.words * sizeof(uint32_t);
        const int64_t blocks64 = (L.T + warps - 1) / warps;
        const int blocks = static_cast<int>(blocks64 < 65536 ? blocks64 : 65536);
        if (L.T > 0) {
            k_bitsets<<<blocks, warps * 32, smem, st>>>(L.sel, L.cu, L.B, L.T, L.Hkv, L.kmax,
                                                        L.words, L.bits, L.counts, L.status);
            if ((e = cudaGetLastError()) != cudaSuccess)
                return e;
        }
    }
    // 2. greedy, one warp per window
    if (L.n_windows > 0) {
        const size_t per_warp = static_cast<size_t>(L.words) * (L.W + 1) * sizeof(uint32_t);
        int warps = static_cast<int>((96 * 1024) / per_warp);
        warps = warps < 1 ? 1 : (warps > 4 ? 4 : warps);
        const size_t smem = per_warp * warps;
        const int kpl = L.W <= 32 ? 1 : L.W <= 64 ? 2 : L.W <= 128 ? 4 : 8;
        const int wpl = L.words <= 32 ? 1 : 2;
        switch (kpl * 10 + wpl) {
        case 11: e = launch_greedy<1, 1>(L, st, warps, smem); break;
        case 12: e = launch_greedy<1, 2>(L, st, warps, smem); break;
        case 21: e = launch_greedy<2, 1>(L, st, warps, smem); break;
        case 22: e = launch_greedy<2, 2>(L, st, warps, smem); break;
        case 41: e = launch_greedy<4, 1>(L, st, warps, smem); break;
        case 42: e = launch_greedy<4, 2>(L, st, warps, smem); break;
        case 81: e = launch_greedy<8, 1>(L, st, warps, smem); break;
        default: e = launch_greedy<8, 2>(L, st, warps, smem); break;
        }
        if (e != cudaSuccess)
            return e;
    }
    // 3. offsets, 4. pages
    k_union_offsets<<<1, 1024, 0, st>>>(L.ucount, L.n_groups, L.union_cap, L.union_off, L.status);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return e;
    if (L.n_groups > 0) {
        const int64_t blocks64 = (L.n_groups + 7) / 8;
        const int blocks = static_cast<int>(blocks64 < 65536 ? blocks64 : 65536);
        k_union_pages<<<blocks, 256, 0, st>>>(L.ubits, L.union_off, L.n_groups, L.words,
                                              L.union_cap, L.union_pages);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

} // namespace pw
