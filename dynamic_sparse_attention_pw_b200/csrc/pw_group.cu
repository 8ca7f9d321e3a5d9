// pw_group.cu -- the bounded GPU search of PageWeaver ("PageWeaver: KV-Guided Query Unions for
// Sparse Attention", Abstract: a bounded GPU search produces query IDs; AI Radio episode on the
// paper, paper summary: greedy inside a bounded window, collecting queries whose selected sets
// add few new pages, with the execution size g fixed independently of W).
//
// Four or five launches on the caller's stream:
//   k_bitsets        sel_pages -> per-(token, kv head) page bitsets + set sizes (validation)
//   k_greedy_local   (long sequences only) one warp per (sequence, kv head, window): the
//                    window's pages renumbered densely, then the ballot/popcount greedy on the
//                    short rows
//   k_greedy<..>     the same greedy on rows of the sequence's length: short sequences, and
//                    the windows whose page union is too large to renumber into 8 words
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
// k_bitsets: one warp per token (grid-stride), hc kv heads at a time.  Lane j reads id j
// (j + 32, ...) of every one of those heads (coalesced rows of kmax ids); the ids are OR-ed
// into per-head bitsets in shared memory and written out as hc contiguous rows.  Invalid ids
// (outside [-1, own page]) are reported and skipped.  counts[t, h] = |S(t, h)| (distinct
// pages).  When one load per lane and head covers a token (kmax <= 32, Hkv <= 8), the next
// token's ids are loaded while the current one is built, and the set sizes are counted as the
// bits are set.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void bitsets_fold(const int32_t *p, int nload, int hh, int own,
                                             int words, uint32_t *acc, int32_t *status)
{
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        if (u >= nload || p[u] == -1)
            continue;
        if (p[u] < -1 || p[u] > own) {
            set_status(status, PW_ERR_BAD_SELECTION);
            continue;
        }
        atomicOr(&acc[(hh + u) * words + (p[u] >> 5)], 1u << (p[u] & 31));
    }
}

__device__ __forceinline__ void bitsets_emit(int64_t t, int h0, int nh, int Hkv, int words,
                                             int lane, const uint32_t *acc,
                                             uint32_t *__restrict__ bits,
                                             uint16_t *__restrict__ counts)
{
    const int nw = nh * words;
    uint32_t *out = bits + (static_cast<size_t>(t) * Hkv + h0) * words;
    for (int i = lane; i < nw; i += 32)
        out[i] = acc[i];
    for (int h = 0; h < nh; ++h) {
        uint32_t cnt = 0;
        for (int w = lane; w < words; w += 32)
            cnt += __popc(acc[h * words + w]);
        cnt = __reduce_add_sync(kFull, cnt);
        if (lane == 0)
            counts[static_cast<size_t>(t) * Hkv + h0 + h] = static_cast<uint16_t>(cnt);
    }
}

__global__ void __launch_bounds__(256) k_bitsets(const int32_t *__restrict__ sel,
                                                 const int32_t *__restrict__ cu, int B, int64_t T,
                                                 int Hkv, int kmax, int words, int hc,
                                                 uint32_t *__restrict__ bits,
                                                 uint16_t *__restrict__ counts, int32_t *status)
{
    constexpr int kLoads = 8;
    extern __shared__ uint32_t sh_acc[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    // per warp: hc bitset rows, then hc set-size counters, rounded up to 16 bytes
    const int region = (hc * words + hc + 3) & ~3;
    uint32_t *acc = sh_acc + wib * region;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + wib;
    if (kmax <= 32 && Hkv <= kLoads) {
        // hc == Hkv here: one pass per token, its ids one load per lane and head.  A set's size
        // is counted as its bits are set (an id whose bit was clear adds one), and the rows go
        // out as 16-byte vectors when they allow it.
        const int nw = Hkv * words;
        uint32_t *cnt = acc + nw;
        const bool vec = (nw & 3) == 0 && (reinterpret_cast<uintptr_t>(bits) & 15) == 0;
        int32_t p[kLoads];
#pragma unroll
        for (int u = 0; u < kLoads; ++u)
            p[u] = t0 < T && u < Hkv && lane < kmax ? sel[(t0 * Hkv + u) * kmax + lane] : -1;
        for (int64_t t = t0; t < T; t += nwarps) {
            const int64_t tn = t + nwarps;
            int32_t q[kLoads];
#pragma unroll
            for (int u = 0; u < kLoads; ++u)
                q[u] = tn < T && u < Hkv && lane < kmax ? sel[(tn * Hkv + u) * kmax + lane] : -1;
            const int b = seq_of_token(cu, B, t);
            const int own = static_cast<int>((t - cu[b]) >> 6);
            if (vec) {
                for (int i = lane; i < (nw >> 2); i += 32)
                    reinterpret_cast<uint4 *>(acc)[i] = make_uint4(0u, 0u, 0u, 0u);
            } else {
                for (int i = lane; i < nw; i += 32)
                    acc[i] = 0;
            }
            if (lane < Hkv)
                cnt[lane] = 0;
            __syncwarp();
#pragma unroll
            for (int u = 0; u < kLoads; ++u) {
                if (u >= Hkv || p[u] == -1)
                    continue;
                if (p[u] < -1 || p[u] > own) {
                    set_status(status, PW_ERR_BAD_SELECTION);
                    continue;
                }
                const uint32_t bit = 1u << (p[u] & 31);
                if ((atomicOr(&acc[u * words + (p[u] >> 5)], bit) & bit) == 0u)
                    atomicAdd(&cnt[u], 1u);
            }
            __syncwarp();
            uint32_t *out = bits + static_cast<size_t>(t) * nw;
            if (vec) {
                for (int i = lane; i < (nw >> 2); i += 32)
                    reinterpret_cast<uint4 *>(out)[i] = reinterpret_cast<const uint4 *>(acc)[i];
            } else {
                for (int i = lane; i < nw; i += 32)
                    out[i] = acc[i];
            }
            if (lane < Hkv)
                counts[static_cast<size_t>(t) * Hkv + lane] = static_cast<uint16_t>(cnt[lane]);
            __syncwarp();
#pragma unroll
            for (int u = 0; u < kLoads; ++u)
                p[u] = q[u];
        }
        return;
    }
    for (int64_t t = t0; t < T; t += nwarps) {
        const int b = seq_of_token(cu, B, t);
        const int own = static_cast<int>((t - cu[b]) >> 6);
        for (int h0 = 0; h0 < Hkv; h0 += hc) {
            const int nh = min(hc, Hkv - h0);
            for (int i = lane; i < nh * words; i += 32)
                acc[i] = 0;
            __syncwarp();
            const int32_t *row = sel + (static_cast<size_t>(t) * Hkv + h0) * kmax;
            for (int j = lane; j - lane < kmax; j += 32) {
                for (int hh = 0; hh < nh; hh += kLoads) {
                    int32_t p[kLoads];
#pragma unroll
                    for (int u = 0; u < kLoads; ++u)
                        p[u] = j < kmax && hh + u < nh ? row[(hh + u) * kmax + j] : -1;
                    bitsets_fold(p, min(kLoads, nh - hh), hh, own, words, acc, status);
                }
            }
            __syncwarp();
            bitsets_emit(t, h0, nh, Hkv, words, lane, acc, bits, counts);
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

// The greedy over one window of n candidates whose bitsets sit in shared memory, transposed:
// sb[w * stride + c] is word w (< nw) of candidate c's set.  Lane l owns candidates l, l + 32,
// ... (KPL of them) and union words l, l + 32, ... (WPL of them).  Costs are maintained
// incrementally:
//   at a seed:  cost(c) = |S(c)| - |S(c) & S(seed)|
//   at a pick:  cost(c) -= |S(c) & (S(pick) \ U)|   and U |= S(pick)
// which equals |S(c) \ U| at every step.  argmin(cost, index) is one redux.sync.min over the
// packed key (cost << 16 | index), so ties go to the lowest token index.  The picks depend on
// set sizes and overlaps only, so any one-to-one renumbering of the pages in sb gives the
// same groups.  For each group, emit(memb, m, U) gets the members (bit k of lane l: candidate
// l + 32 k), the group size and the union words in sb's numbering.
template <int KPL, int WPL, class Emit>
__device__ __forceinline__ void greedy_window(const uint32_t *sb, int stride, int nw, int n,
                                              const int (&cnt)[KPL], int g, int lane, Emit &emit)
{
    uint32_t avail = 0;
#pragma unroll
    for (int k = 0; k < KPL; ++k)
        if (lane + 32 * k < n)
            avail |= 1u << k;
    int remaining = n;
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
            U[j] = w < nw ? sb[w * stride + seed] : 0u;
        }
        int cost[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k)
            cost[k] = cnt[k];
        if (g > 1 && remaining > 0)
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
                const uint32_t s = w < nw ? sb[w * stride + c] : 0u;
                Dlt[j] = s & ~U[j];
                U[j] |= s;
            }
            subtract_overlap<KPL, WPL>(Dlt, sb, stride, lane, avail, cost);
        }
        emit(memb, m, U);
    }
}

// Writes group gidx of window win: members ascending (candidate index = lane + 32 k, so
// k-major then lane), -1 padding, the union bitset (lane l holds word l + 32 j in U[j]; words
// past the sequence's are zero), its size and the group's (b, h, w).
template <int KPL, int WPL>
__device__ __forceinline__ void write_group(const Window &win, int64_t gidx, uint32_t memb, int m,
                                            const uint32_t (&U)[WPL], int g, int words, int lane,
                                            int32_t *qids, int32_t *gsize, int32_t *gmeta,
                                            uint32_t *ubits, int32_t *ucount)
{
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
}

// Bitset words that can be non-zero in window win: a token selects no page after its own
// (later ids are rejected by k_bitsets), so no page past the last token's own page.
__device__ __forceinline__ int window_words(const Window &win, int W)
{
    const int last_page = (win.w * W + win.n - 1) >> 6;
    return min(win.nwb, (last_page >> 5) + 1);
}

// ---------------------------------------------------------------------------------------
// k_greedy: one warp per window, the window's bitsets staged in shared memory transposed
// ([word][candidate], stride W + 1, so that lanes owning consecutive candidates read
// consecutive words).  With deferred_only it takes only the windows k_greedy_local left to
// it (gsize of their first group -1) and skips the rest.  Warps take the windows from the
// last one down: the later windows of a sequence, and the longer sequences, cost the most,
// so they start first.
// ---------------------------------------------------------------------------------------
template <int KPL, int WPL>
__global__ void __launch_bounds__(128) k_greedy(
    const uint32_t *__restrict__ bits, const uint16_t *__restrict__ counts,
    const int32_t *__restrict__ cu, int B, int Hkv, int words, int W, int g,
    int64_t n_windows, int deferred_only, int32_t *__restrict__ qids,
    int32_t *__restrict__ gsize, int32_t *__restrict__ gmeta, uint32_t *__restrict__ ubits,
    int32_t *__restrict__ ucount)
{
    extern __shared__ uint32_t sh_win[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int stride = W + 1;
    uint32_t *sb = sh_win + static_cast<size_t>(wib) * words * stride;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);

    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + wib;
         wi < n_windows; wi += nwarps) {
        const Window win = locate_window(n_windows - 1 - wi, cu, B, Hkv, W, g);
        if (deferred_only && gsize[win.gbase] != -1)
            continue;
        const int n = win.n, nww = window_words(win, W);
        const int total = n * nww;
        for (int q = lane; q < total; q += 32) {
            const int c = q / nww, w = q - c * nww;
            sb[w * stride + c] =
                bits[(static_cast<size_t>(win.tok0 + c) * Hkv + win.h) * words + w];
        }
        int cnt[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int c = lane + 32 * k;
            cnt[k] = c < n ? counts[static_cast<size_t>(win.tok0 + c) * Hkv + win.h] : 0;
        }
        __syncwarp();
        int64_t gidx = win.gbase;
        auto emit = [&](uint32_t memb, int m, const uint32_t (&U)[WPL]) {
            write_group<KPL, WPL>(win, gidx, memb, m, U, g, words, lane, qids, gsize, gmeta,
                                  ubits, ucount);
            ++gidx;
        };
        greedy_window<KPL, WPL>(sb, stride, nww, n, cnt, g, lane, emit);
        __syncwarp();
    }
}

// Bit r of the result is set when v holds the r-th set bit of mask (v a subset of mask).
__device__ __forceinline__ uint32_t gather_bits(uint32_t v, uint32_t mask)
{
    if (mask == kFull)
        return v;
    uint32_t r = 0;
    while (v) {
        const int b = __ffs(v) - 1;
        v &= v - 1;
        r |= 1u << __popc(mask & ((1u << b) - 1u));
    }
    return r;
}

// The inverse of gather_bits: bit r of f goes to the position of the r-th set bit of mask.
__device__ __forceinline__ uint32_t scatter_bits(uint32_t f, uint32_t mask)
{
    if (mask == kFull)
        return f;
    uint32_t r = 0;
    while (f) {
        const uint32_t low = mask & (0u - mask);
        if (f & 1u)
            r |= low;
        mask ^= low;
        f >>= 1;
    }
    return r;
}

// Renumbering one candidate's set: the lane's global words v[j] give renumbered bit fields
// lo[j] (in local word wlo[j]) and hi[j] (in local word wlo[j] + 1).
template <int WPL>
__device__ __forceinline__ void renumber_parts(const uint32_t (&v)[WPL], const uint32_t (&P)[WPL],
                                               const int (&base)[WPL], uint32_t (&lo)[WPL],
                                               uint32_t (&hi)[WPL], int (&wlo)[WPL])
{
#pragma unroll
    for (int j = 0; j < WPL; ++j) {
        const uint32_t f = gather_bits(v[j], P[j]);
        const int sh = base[j] & 31;
        wlo[j] = base[j] >> 5;
        lo[j] = f << sh;
        hi[j] = sh ? f >> (32 - sh) : 0u;
    }
}

// Local word x of the candidate's renumbered set: the OR of every lane's part of it.
template <int WPL>
__device__ __forceinline__ uint32_t local_word(const uint32_t (&lo)[WPL], const uint32_t (&hi)[WPL],
                                               const int (&wlo)[WPL], int x)
{
    uint32_t part = 0;
#pragma unroll
    for (int j = 0; j < WPL; ++j)
        part |= (wlo[j] == x ? lo[j] : 0u) | (wlo[j] + 1 == x ? hi[j] : 0u);
    return __reduce_or_sync(kFull, part);
}

// Word (lane, j) of a renumbered set in page ids: the field of local bits [base, base + |P|),
// taken from local words a (= base / 32) and b (the next one), scattered onto P's set bits.
__device__ __forceinline__ uint32_t to_page_ids(uint32_t a, uint32_t b, uint32_t P, int base)
{
    const int sh = base & 31, cw = __popc(P);
    uint32_t f = sh ? (a >> sh) | (b << (32 - sh)) : a;
    f &= cw >= 32 ? kFull : ((1u << cw) - 1u);
    return scatter_bits(f, P);
}

// The greedy of k_greedy for a renumbered window whose sets fit LW local words, held in
// registers: R[k][x] is local word x of candidate lane + 32 k.  A seed's or a pick's set
// reaches every lane by LW shuffles, the union U is kept whole in every lane, and a cost
// update is LW popcounts per candidate, with no shared-memory round trip on the chain from
// one pick to the next.
template <int KPL, int WPL, int LW>
__device__ __forceinline__ void greedy_window_regs(
    const Window &win, const uint32_t *rows, size_t rstride, int nww, const uint32_t (&P)[WPL],
    const int (&base)[WPL], const int (&cnt)[KPL], int g, int words, int lane, uint32_t *wsm,
    int32_t *qids, int32_t *gsize, int32_t *gmeta, uint32_t *ubits, int32_t *ucount)
{
    constexpr int kRows = 8 / WPL;
    constexpr int TS = 32 * WPL + 1; // tile row stride, odd: conflict-free by rows and by columns
    const int n = win.n;
    uint32_t *tile = wsm;
    const uint32_t *Psh = wsm + 32 * TS;
    const int32_t *Bsh = reinterpret_cast<const int32_t *>(Psh + 32 * WPL);
    // Renumbering, 32 candidates at a time: their rows pass through the tile (lane = word on
    // the way in, lane = candidate on the way out), and lane r folds candidate 32 k + r's
    // words, each gathered onto its word's local numbers, into R[k].
    uint32_t R[KPL][LW];
#pragma unroll
    for (int k = 0; k < KPL; ++k) {
#pragma unroll
        for (int x = 0; x < LW; ++x)
            R[k][x] = 0u;
        if (32 * k >= n)
            continue;
        for (int r0 = 0; r0 < 32; r0 += kRows) {
            const int c0 = 32 * k + r0;
            uint32_t v[kRows][WPL];
#pragma unroll
            for (int u = 0; u < kRows; ++u)
#pragma unroll
                for (int j = 0; j < WPL; ++j) {
                    const int w = lane + 32 * j;
                    v[u][j] = c0 + u < n && w < nww ? rows[(c0 + u) * rstride + w] : 0u;
                }
#pragma unroll
            for (int u = 0; u < kRows; ++u)
#pragma unroll
                for (int j = 0; j < WPL; ++j)
                    tile[(r0 + u) * TS + lane + 32 * j] = v[u][j];
        }
        __syncwarp();
        for (int w = 0; w < nww; ++w) {
            const uint32_t f = gather_bits(tile[lane * TS + w], Psh[w]);
            const int bw = Bsh[w], x0 = bw >> 5, sh = bw & 31;
            const uint32_t lo = f << sh, hi = sh ? f >> (32 - sh) : 0u;
#pragma unroll
            for (int x = 0; x < LW; ++x)
                R[k][x] |= (x == x0 ? lo : 0u) | (x == x0 + 1 ? hi : 0u);
        }
        __syncwarp();
    }

    // key[k] = cost << 16 | index of candidate lane + 32 k while it is available, near ~0
    // once taken or absent (costs stay below 2^8 here, and the ~0 of a taken candidate loses
    // less than 2^8 << 16 over a group, so it never wins a pick)
    uint32_t avail = 0;
#pragma unroll
    for (int k = 0; k < KPL; ++k)
        if (lane + 32 * k < n)
            avail |= 1u << k;
    int remaining = n;
    int64_t gidx = win.gbase;
    while (remaining > 0) {
        uint32_t mine = 0xFFFFFFFFu;
#pragma unroll
        for (int k = KPL - 1; k >= 0; --k)
            if ((avail >> k) & 1u)
                mine = lane + 32 * k;
        uint32_t c = __reduce_min_sync(kFull, mine);
        uint32_t memb = 0;
        int m = 0;
        uint32_t U[LW];
#pragma unroll
        for (int x = 0; x < LW; ++x)
            U[x] = 0u;
        uint32_t key[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k)
            key[k] = (avail >> k) & 1u ? (static_cast<uint32_t>(cnt[k]) << 16) |
                                             static_cast<uint32_t>(lane + 32 * k)
                                       : 0xFFFFFFFFu;
        // the seed, then each pick: take c, add its new pages to U, charge them to the rest
        for (;;) {
            const int slot = static_cast<int>(c >> 5), src = static_cast<int>(c & 31u);
            if (src == lane) {
                avail &= ~(1u << slot);
                memb |= 1u << slot;
#pragma unroll
                for (int k = 0; k < KPL; ++k)
                    key[k] = k == slot ? 0xFFFFFFFFu : key[k];
            }
            --remaining;
            ++m;
            uint32_t d[LW];
#pragma unroll
            for (int x = 0; x < LW; ++x) {
                uint32_t t = R[0][x];
#pragma unroll
                for (int k = 1; k < KPL; ++k)
                    t = slot == k ? R[k][x] : t;
                const uint32_t sx = __shfl_sync(kFull, t, src);
                d[x] = sx & ~U[x];
                U[x] |= sx;
            }
            if (m >= g || remaining <= 0)
                break;
            uint32_t any = 0;
#pragma unroll
            for (int x = 0; x < LW; ++x)
                any |= d[x];
            if (any) { // the same in every lane
#pragma unroll
                for (int k = 0; k < KPL; ++k) {
                    uint32_t pc = 0;
#pragma unroll
                    for (int x = 0; x < LW; ++x)
                        pc += __popc(R[k][x] & d[x]);
                    key[k] -= pc << 16;
                }
            }
            uint32_t kmin = key[0];
#pragma unroll
            for (int k = 1; k < KPL; ++k)
                kmin = min(kmin, key[k]);
            c = __reduce_min_sync(kFull, kmin) & 0xFFFFu;
        }
        uint32_t Ug[WPL];
#pragma unroll
        for (int j = 0; j < WPL; ++j) {
            const int wl = base[j] >> 5;
            uint32_t a = 0u, b = 0u;
#pragma unroll
            for (int x = 0; x < LW; ++x) {
                a = x == wl ? U[x] : a;
                b = x == wl + 1 ? U[x] : b;
            }
            Ug[j] = to_page_ids(a, b, P[j], base[j]);
        }
        write_group<KPL, WPL>(win, gidx, memb, m, Ug, g, words, lane, qids, gsize, gmeta, ubits,
                              ucount);
        ++gidx;
    }
}

// ---------------------------------------------------------------------------------------
// k_greedy_local: one warp per window, the window's pages renumbered before the search.  The
// union P of the window's sets (lane l holds words l + 32 j) numbers each of its pages by its
// rank in P; every candidate's set is rewritten in those local numbers, so that the staged
// rows, and the words each seed and pick visits, number ceil(|P| / 32) instead of the
// sequence's.  The search itself is k_greedy's (the renumbering is one-to-one), and each
// group's union goes back to page ids before it is written.  Sets of up to four local words
// stay in registers (greedy_window_regs); up to lw words they are staged in shared memory; a
// window whose union holds more than 32 lw pages is left to k_greedy: gsize of its first
// group is set to -1.
// ---------------------------------------------------------------------------------------
template <int KPL, int WPL>
__global__ void __launch_bounds__(128) k_greedy_local(
    const uint32_t *__restrict__ bits, const uint16_t *__restrict__ counts,
    const int32_t *__restrict__ cu, int B, int Hkv, int words, int W, int g, int lw, int wsz,
    int64_t n_windows, int32_t *__restrict__ qids, int32_t *__restrict__ gsize,
    int32_t *__restrict__ gmeta, uint32_t *__restrict__ ubits, int32_t *__restrict__ ucount)
{
    constexpr int kRows = 8 / WPL; // candidate rows in flight per lane
    extern __shared__ uint32_t sh_win[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int stride = W + 1;
    // the warp's wsz words: the renumbering tile and the words' local numbering (register
    // paths), or the staged rows sb (more than four local words)
    uint32_t *sb = sh_win + static_cast<size_t>(wib) * wsz;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const size_t rstride = static_cast<size_t>(Hkv) * words;

    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + wib;
         wi < n_windows; wi += nwarps) {
        const Window win = locate_window(n_windows - 1 - wi, cu, B, Hkv, W, g);
        const int n = win.n, nww = window_words(win, W);
        const uint32_t *rows = bits + (static_cast<size_t>(win.tok0) * Hkv + win.h) * words;

        // 1. the window's page union
        uint32_t P[WPL];
#pragma unroll
        for (int j = 0; j < WPL; ++j)
            P[j] = 0u;
        for (int c0 = 0; c0 < n; c0 += kRows) {
            uint32_t v[kRows][WPL];
#pragma unroll
            for (int u = 0; u < kRows; ++u)
#pragma unroll
                for (int j = 0; j < WPL; ++j) {
                    const int w = lane + 32 * j;
                    v[u][j] = c0 + u < n && w < nww ? rows[(c0 + u) * rstride + w] : 0u;
                }
#pragma unroll
            for (int u = 0; u < kRows; ++u)
#pragma unroll
                for (int j = 0; j < WPL; ++j)
                    P[j] |= v[u][j];
        }
        // local number of the first page of word (lane, j): the pages of the words before it
        int base[WPL];
        int nloc = 0;
#pragma unroll
        for (int j = 0; j < WPL; ++j) {
            const int c = __popc(P[j]);
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int x = __shfl_up_sync(kFull, incl, off);
                if (lane >= off)
                    incl += x;
            }
            base[j] = nloc + incl - c;
            nloc += __shfl_sync(kFull, incl, 31);
        }
        if (nloc > 32 * lw) {
            if (lane == 0)
                gsize[win.gbase] = -1;
            continue;
        }
        const int nlw = (nloc + 31) >> 5;
        int cnt[KPL];
#pragma unroll
        for (int k = 0; k < KPL; ++k) {
            const int c = lane + 32 * k;
            cnt[k] = c < n ? counts[static_cast<size_t>(win.tok0 + c) * Hkv + win.h] : 0;
        }
        if (nlw <= 4) {
            uint32_t *Psh = sb + 32 * (32 * WPL + 1);
#pragma unroll
            for (int j = 0; j < WPL; ++j) {
                Psh[lane + 32 * j] = P[j];
                Psh[32 * WPL + lane + 32 * j] = static_cast<uint32_t>(base[j]);
            }
            if (nlw <= 2)
                greedy_window_regs<KPL, WPL, 2>(win, rows, rstride, nww, P, base, cnt, g, words,
                                                lane, sb, qids, gsize, gmeta, ubits, ucount);
            else
                greedy_window_regs<KPL, WPL, 4>(win, rows, rstride, nww, P, base, cnt, g, words,
                                                lane, sb, qids, gsize, gmeta, ubits, ucount);
            __syncwarp();
            continue;
        }

        // 2. more than four local words: each candidate's set in local numbers ->
        // sb[x * stride + c], lane x < nlw storing local word x
        for (int c0 = 0; c0 < n; c0 += kRows) {
            uint32_t v[kRows][WPL];
#pragma unroll
            for (int u = 0; u < kRows; ++u)
#pragma unroll
                for (int j = 0; j < WPL; ++j) {
                    const int w = lane + 32 * j;
                    v[u][j] = c0 + u < n && w < nww ? rows[(c0 + u) * rstride + w] : 0u;
                }
#pragma unroll
            for (int u = 0; u < kRows; ++u) {
                if (c0 + u >= n)
                    break;
                uint32_t lo[WPL], hi[WPL];
                int wlo[WPL];
                renumber_parts<WPL>(v[u], P, base, lo, hi, wlo);
                uint32_t mine = 0;
                for (int x = 0; x < nlw; ++x) {
                    const uint32_t r = local_word<WPL>(lo, hi, wlo, x);
                    if (lane == x)
                        mine = r;
                }
                if (lane < nlw)
                    sb[lane * stride + c0 + u] = mine;
            }
        }
        __syncwarp();

        int64_t gidx = win.gbase;
        auto emit = [&](uint32_t memb, int m, const uint32_t (&Ul)[1]) {
            uint32_t Ug[WPL];
#pragma unroll
            for (int j = 0; j < WPL; ++j) {
                const int wl = base[j] >> 5;
                const uint32_t a = __shfl_sync(kFull, Ul[0], wl & 31);
                const uint32_t b = __shfl_sync(kFull, Ul[0], (wl + 1) & 31);
                Ug[j] = to_page_ids(a, b, P[j], base[j]);
            }
            write_group<KPL, WPL>(win, gidx, memb, m, Ug, g, words, lane, qids, gsize, gmeta,
                                  ubits, ucount);
            ++gidx;
        };
        greedy_window<KPL, 1>(sb, stride, nlw, n, cnt, g, lane, emit);
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------------------
// k_union_offsets: single block; exclusive scan of ucount -> union_off[0..n].  Warp v owns
// the contiguous range [v c, (v + 1) c), c a multiple of 128, which it walks 128 entries at a
// time (lane l: entries 4 l .. 4 l + 3, one int4 where both arrays are 16-byte aligned), so
// that every load and store of a warp is one contiguous 512-byte run: one pass for the warp
// sums, a block scan of the sums, one pass for the offsets.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int4 load4(const int32_t *p, int64_t i, int64_t n, bool vec)
{
    if (vec && i + 3 < n)
        return *reinterpret_cast<const int4 *>(p + i);
    return make_int4(i < n ? p[i] : 0, i + 1 < n ? p[i + 1] : 0, i + 2 < n ? p[i + 2] : 0,
                     i + 3 < n ? p[i + 3] : 0);
}

__global__ void __launch_bounds__(1024) k_union_offsets(const int32_t *__restrict__ ucount,
                                                        int64_t n, int64_t cap,
                                                        int32_t *__restrict__ union_off,
                                                        int32_t *status)
{
    constexpr int kVec = 4; // 128-entry steps in flight per warp
    __shared__ long long wsum[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
    const int64_t per = 128 * kVec;
    const int64_t chunk = (n + static_cast<int64_t>(nwarp) * per - 1) / (static_cast<int64_t>(nwarp) * per) * per;
    const int64_t s = min(n, static_cast<int64_t>(warp) * chunk);
    const int64_t e = min(n, s + chunk);
    const bool vec = ((reinterpret_cast<uintptr_t>(ucount) | reinterpret_cast<uintptr_t>(union_off)) & 15) == 0;
    long long local = 0;
    for (int64_t i0 = s; i0 < e; i0 += per) {
        int4 v[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u)
            v[u] = load4(ucount, i0 + 128 * u + 4 * lane, e, vec);
#pragma unroll
        for (int u = 0; u < kVec; ++u)
            local += static_cast<long long>(v[u].x) + v[u].y + v[u].z + v[u].w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        local += __shfl_xor_sync(kFull, local, off);
    if (lane == 0)
        wsum[warp] = local;
    __syncthreads();
    if (warp == 0) {
        long long v = lane < nwarp ? wsum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long u = __shfl_up_sync(kFull, v, off);
            if (lane >= off)
                v += u;
        }
        if (lane < nwarp)
            wsum[lane] = v;
    }
    __syncthreads();
    long long base = warp > 0 ? wsum[warp - 1] : 0;
    for (int64_t i0 = s; i0 < e; i0 += per) {
        int4 v[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u)
            v[u] = load4(ucount, i0 + 128 * u + 4 * lane, e, vec);
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int64_t i = i0 + 128 * u + 4 * lane;
            const long long t4 = static_cast<long long>(v[u].x) + v[u].y + v[u].z + v[u].w;
            long long incl = t4;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long x = __shfl_up_sync(kFull, incl, off);
                if (lane >= off)
                    incl += x;
            }
            const long long b0 = base + incl - t4;
            const int4 o = make_int4(static_cast<int32_t>(b0), static_cast<int32_t>(b0 + v[u].x),
                                     static_cast<int32_t>(b0 + v[u].x + v[u].y),
                                     static_cast<int32_t>(b0 + v[u].x + v[u].y + v[u].z));
            if (vec && i + 3 < e) {
                *reinterpret_cast<int4 *>(union_off + i) = o;
            } else {
                if (i < e)
                    union_off[i] = o.x;
                if (i + 1 < e)
                    union_off[i + 1] = o.y;
                if (i + 2 < e)
                    union_off[i + 2] = o.z;
                if (i + 3 < e)
                    union_off[i + 3] = o.w;
            }
            base += __shfl_sync(kFull, incl, 31);
        }
    }
    if (tid == 0) {
        const long long total = wsum[nwarp - 1];
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
cudaError_t launch_greedy(const GroupLaunch &L, cudaStream_t st, int lw)
{
    const int warps = 4;
    if (lw > 0) {
        // renumbered windows first
        auto kern = k_greedy_local<KPL, WPL>;
        const int tile_words = 32 * (32 * WPL + 1) + 64 * WPL, rows_words = lw * (L.W + 1);
        const int wsz = tile_words > rows_words ? tile_words : rows_words;
        const size_t smem = static_cast<size_t>(wsz) * sizeof(uint32_t) * warps;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        const int64_t blocks64 = (L.n_windows + warps - 1) / warps;
        const int blocks = static_cast<int>(blocks64 < 1048576 ? blocks64 : 1048576);
        kern<<<blocks, warps * 32, smem, st>>>(L.bits, L.counts, L.cu, L.B, L.Hkv, L.words, L.W,
                                               L.g, lw, wsz, L.n_windows, L.qids, L.gsize,
                                               L.gmeta, L.ubits, L.ucount);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    // the sequence's words staged in shared memory: every window, or (after k_greedy_local)
    // the ones it left, whose warps do the work while the others return at once
    auto kern = k_greedy<KPL, WPL>;
    const size_t per_warp = static_cast<size_t>(L.words) * (L.W + 1) * sizeof(uint32_t);
    int gwarps = static_cast<int>((96 * 1024) / per_warp);
    gwarps = gwarps < 1 ? 1 : (gwarps > warps ? warps : gwarps);
    const size_t smem = per_warp * gwarps;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    const int64_t blocks64 = (L.n_windows + gwarps - 1) / gwarps;
    const int blocks = static_cast<int>(blocks64 < 1048576 ? blocks64 : 1048576);
    kern<<<blocks, gwarps * 32, smem, st>>>(L.bits, L.counts, L.cu, L.B, L.Hkv, L.words, L.W, L.g,
                                            L.n_windows, lw > 0 ? 1 : 0, L.qids, L.gsize, L.gmeta,
                                            L.ubits, L.ucount);
    return cudaGetLastError();
}

} // namespace

cudaError_t group_launch(const GroupLaunch &L, cudaStream_t st)
{
    cudaError_t e;
    // 1. bitsets
    {
        const int warps = 8;
        int hc = 512 / L.words; // heads per pass: at most 2 KiB of bitsets per warp
        hc = hc < 1 ? 1 : (hc > L.Hkv ? L.Hkv : hc);
        const size_t smem = static_cast<size_t>(warps) * ((hc * L.words + hc + 3) & ~3) *
                            sizeof(uint32_t);
        // one resident wave of warps striding over the tokens (each warp prefetches its next
        // token's ids)
        int dev = 0, sms = 0, per_sm = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_bitsets, warps * 32,
                                                               smem)) != cudaSuccess)
            return e;
        const int64_t wave = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
        int64_t blocks64 = (L.T + warps - 1) / warps;
        blocks64 = blocks64 < wave ? blocks64 : wave;
        const int blocks = static_cast<int>(blocks64);
        if (L.T > 0) {
            k_bitsets<<<blocks, warps * 32, smem, st>>>(L.sel, L.cu, L.B, L.T, L.Hkv, L.kmax,
                                                        L.words, hc, L.bits, L.counts, L.status);
            if ((e = cudaGetLastError()) != cudaSuccess)
                return e;
        }
    }
    // 2. greedy, one warp per window.  Windows are renumbered first (k_greedy_local) when their
    // rows staged whole would take more than about 8 KiB of shared memory per warp, which
    // would leave too few warps per SM; otherwise they are staged as they are.
    if (L.n_windows > 0) {
        constexpr int kLocalWords = 8, kStagedWordsPerWarp = 2112;
        const int lw = L.words > kLocalWords && L.words * (L.W + 1) > kStagedWordsPerWarp
                           ? kLocalWords : 0;
        const int kpl = L.W <= 32 ? 1 : L.W <= 64 ? 2 : L.W <= 128 ? 4 : 8;
        const int wpl = L.words <= 32 ? 1 : 2;
        switch (kpl * 10 + wpl) {
        case 11: e = launch_greedy<1, 1>(L, st, lw); break;
        case 12: e = launch_greedy<1, 2>(L, st, lw); break;
        case 21: e = launch_greedy<2, 1>(L, st, lw); break;
        case 22: e = launch_greedy<2, 2>(L, st, lw); break;
        case 41: e = launch_greedy<4, 1>(L, st, lw); break;
        case 42: e = launch_greedy<4, 2>(L, st, lw); break;
        case 81: e = launch_greedy<8, 1>(L, st, lw); break;
        default: e = launch_greedy<8, 2>(L, st, lw); break;
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
