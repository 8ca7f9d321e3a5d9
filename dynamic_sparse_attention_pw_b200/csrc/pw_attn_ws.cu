// pw_attn_ws.cu -- persistent, warp-specialised ID-aware union attention (tiles of <= 64 rows).
//
// Same result as the one-group-per-CTA kernel in pw_attn.cu ("PageWeaver: KV-Guided Query
// Unions for Sparse Attention", Abstract: union pages loaded once per group, each query masked
// to its own support, complete output per query, FP8 KV), organised so that the tensor-core
// work of one page overlaps the decode and softmax work of its neighbours.
//
// S = Q K^T runs on the FP8 tensor-core path with the E4M3 K page exactly as stored: each Q row
// is scaled by a power of two and split into two E4M3 parts, q' = q1 + q2, which is exact for
// every element within 2^9 of the row's largest (an 8-bit bf16 significand is a 4-bit E4M3
// significand plus a remainder of at most 4 bits); S = (q1 K^T + q2 K^T) 2^-s.  The product
// O += P V runs on f16 operands with P read from TMEM: P split into f16 hi + lo parts, both
// multiplied into the one accumulator, and V decoded exactly (E4M3 is a subset of f16).
//
// One CTA per SM walks the groups blockIdx.x, blockIdx.x + gridDim.x, ... (a ragged batch: takes
// them from a work counter, the last group first, until none are left).  A step is one or two
// union pages of a group.  Its warps:
//   warps 0-3    decode   E4M3 V pages -> f16 operand tiles, one step at a time
//   warps 4-11   softmax  S -> P for each step (four threads per row, 16 keys of each page each;
//                         both pages' scores in one TMEM round trip), written back to TMEM over
//                         the S it came from; lazy O rescale (out of line); per-row sums
//   warps 12-15  epilogue Q tile of the next group (scaled, split into two E4M3 parts) while
//                         the current one runs, then O of the finished group -> bf16 rows of O
//                         (one warp per TMEM lane quadrant)
//   warp 16      load     one group ahead: group records (rows, positions, first membership
//                         words, first page ids), the next group's Q rows by TMA, and the union
//                         pages: K through a tensor map with the 128-byte swizzle the MMA reads,
//                         V by bulk copy
//   warp 17      MMA (S)  S (FP8, N = 64 per page) of each step, up to three steps ahead of
//                         the products
//   warp 18      MMA (PV) O += P V of each step
// Few warps on purpose: the MMA warps sit on the critical path, and every extra busy warp on
// their schedulers delays their waits and issues.  Compact code on purpose too: five roles run
// different code on each scheduler, and on most SMs the kernel slows down in proportion to its
// code size, so cold paths stay out of line or rolled and each role's loop calls each of its
// steps from one place.
// TMEM holds three S/P buffers and one O buffer (M = 64 layout: row r at lane
// 32 (r / 16) + r % 16).  The P of a step replaces its S in place, as the A operand of the products
// (keys 2j and 2j + 1 of a 16-key block packed in column j: P_hi in a block's first 8 columns,
// P_lo in the next 8).  S and the products are issued by two warps, so that neither stream's
// waits hold up the other: S runs up to three steps ahead, as far as the buffers allow.
// Hand-offs per step, all mbarriers: S done (also frees the step's K stage pair), P written and V
// tiles decoded (one barrier), products done (frees the S/P buffer for S three steps later and
// the V step slot for the tiles two steps later).  The first products of a group wait until the
// epilogue has read the previous group's O.  Every wait is bounded and, when it runs out, sets an
// abort flag that releases the other roles.
#include <cstdint>
#include <cuda.h> // CUtensorMap and its enums (the encoder itself is fetched at run time)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "pw_attn_common.cuh"
#include "pw_internal.h"
#include "pw_sm100.cuh"

namespace pw {
namespace {

using namespace attn;

constexpr int kNS = 3;        // S/P buffers in TMEM, one step each
constexpr int kNKP = kNS;     // E4M3 K stage pairs (one S step each), paired with the S buffers
constexpr int kNSV = 4;       // E4M3 V page stages
constexpr int kNJ = 3;        // group records in flight
constexpr int kDecThreads = 128;
constexpr int kSmThreads = 256;
constexpr int kEpiThreads = 128;
constexpr int kWarpSm0 = kDecThreads / 32, kWarpEpi0 = kWarpSm0 + 8, kWarpLoad = kWarpEpi0 + 4,
              kWarpMma = kWarpLoad + 1, kWarpPv = kWarpMma + 1;
constexpr int kThreads = 32 * (kWarpPv + 1);
static_assert(kWarpSm0 % 4 == 0, "softmax warp w must sit in TMEM lane quadrant w % 4");
static_assert(kWarpEpi0 % 4 == 0, "epilogue warp e must sit in TMEM lane quadrant e");
static_assert(kNKP == kNS, "a K stage pair is freed by the S completion of its S buffer");
constexpr uint32_t kTmemCols = 512; // S / P [0..2] at columns 0 / 128 / 256, O at 384
constexpr uint32_t kColS = 128;     // one S step: two pages of 64 keys
constexpr uint32_t kColO = kColS * kNS;
static_assert(kColO + 128 <= kTmemCols, "S/P buffers and O must fit in TMEM");
constexpr uint32_t kFull = 0xFFFFFFFFu;

// One group as the load warp hands it to the other roles, so that none of them meets a chain
// of dependent global loads when it starts a group.
struct GroupJob {
    int32_t tok[64];    // query token of each tile row (rows >= R: 0)
    int32_t pos[64];    // its position within its sequence
    int32_t qexp[64];   // its Q scale exponent (written by the epilogue warps with the Q tile)
    uint32_t word0[2][32]; // per query: its membership words of the first two union pages
    int32_t b, h, R, nU, u0, pg0, pg1, pg2, pg3; // union pages 0..3 (absent ones: pg0); nU < 0: no further group
};

struct __align__(1024) WsSmem {
    uint8_t q[2][2][64 * 128];    // [Q buffer][part q1 / q2][64 rows][128 dims] E4M3, swizzled
    uint8_t v[2][2][2][64 * 128]; // [step slot][page of the step][dim-block][64 keys][64 dims] f16, swizzled
    // E4M3 K pages, 128-byte swizzled by the tensor copy; the two pages of a step sit in one
    // pair, so that they form one 128-row operand
    uint8_t stage_k[kNKP][2][kPageBytes];
    uint8_t stage_v[kNSV][kPageBytes]; // E4M3 V pages, row-major
    uint8_t q_raw[64 * 256];           // bf16 Q rows of the next group, row r at 256 r
    GroupJob job[kNJ];
    float qmax[64][4];    // per-row partial maxima exchanged by the row's four threads
    float lsum[2][64][4]; // [group % 2][row][quarter]: per-thread partial row sums of a group
    uint64_t job_full[kNJ], job_empty[kNJ];
    uint64_t qraw_full, qraw_empty;
    uint64_t kst_full[kNKP];
    uint64_t vst_full[kNSV], vst_empty[kNSV];
    // s_done[n % 3]: S of step n complete; this also frees S's K stage pair (pair n % 3)
    uint64_t s_done[kNS];
    // pvs_done[n % 3]: the products of step n complete; this frees S/P buffer n % 3 for S of
    // step n + 3 and the V step slot n % 2 for the tiles of step n + 2
    uint64_t pvs_done[kNS];
    // pv_ready[n % 3]: P of step n written (one arrival per softmax warp) and its f16 V tiles
    // decoded (one per decode warp): everything the products of step n read.  Neither role can
    // arrive for step n + 3 before the products of step n are complete.
    uint64_t pv_ready[kNS];
    uint64_t q_full[2], q_empty[2];
    uint64_t o_full;    // the last product of a group complete (one phase per group)
    uint64_t l_full[2]; // l_full[g % 2]: the row sums of group g published
    uint64_t o_free[2]; // o_free[g % 2]: the epilogue has read O and lsum[g % 2] of group g
    uint64_t drain_bar;
    uint32_t k_issued, v_issued; // steps / pages whose K / V copies the load warp issued
    uint32_t q_issued;           // groups whose Q rows it copied
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t early_exit;
};

// The layout plus the slack for aligning it to 1024 bytes must fit one CTA's shared memory.
static_assert(sizeof(WsSmem) + 1024 <= 227 * 1024, "shared-memory layout too large");

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait that also gives up as soon as another role has aborted.  The abort flag and the
// clock are read once per eight tries, so a spinning thread issues little besides the tries.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int32_t *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    for (;;) {
#pragma unroll 1
        for (int k = 0; k < 8; ++k)
            if (mbar_try_wait(bar, parity))
                return true;
        if (*reinterpret_cast<volatile int32_t *>(abort_flag) != 0)
            return false;
        if (clock64() - t0 > kWaitCycles) {
            *reinterpret_cast<volatile int32_t *>(abort_flag) = 1;
            return false;
        }
    }
}

// wait_bar for the waits outside the per-step loops of the softmax and MMA warps: the first try
// inline, the spin out of line, so that these wait sites add little code.
__device__ __noinline__ bool wait_bar_spin(uint64_t *bar, uint32_t parity, int32_t *abort_flag)
{
    return wait_bar(bar, parity, abort_flag);
}

__device__ __forceinline__ bool wait_bar_c(uint64_t *bar, uint32_t parity, int32_t *abort_flag)
{
    return mbar_try_wait(bar, parity) || wait_bar_spin(bar, parity, abort_flag);
}

// wait_bar for roles off the critical path (load, epilogue): between tries the thread sleeps,
// so a long wait takes few issue slots from the warps that share its scheduler.
__device__ __noinline__ bool wait_bar_lazy(uint64_t *bar, uint32_t parity, int32_t *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    for (;;) {
        __nanosleep(128);
        if (mbar_try_wait(bar, parity))
            return true;
        if (*reinterpret_cast<volatile int32_t *>(abort_flag) != 0)
            return false;
        if (clock64() - t0 > kWaitCycles) {
            *reinterpret_cast<volatile int32_t *>(abort_flag) = 1;
            return false;
        }
    }
}

// Named barriers (0 is __syncthreads): the epilogue role has one; the softmax
// role has one per TMEM lane quadrant (kBarSoftmax0 + quadrant), shared by the two warps that
// hold that quadrant's rows, so that the quadrants never wait for one another.
constexpr uint32_t kBarEpilogue = 3, kBarSoftmax0 = 4;
constexpr uint32_t kSmQuadThreads = 64;

// Named barrier `id` over `n` threads, returning whether any of them passed `pred`.  Warps
// blocked here issue nothing, so one thread of a role waits on an mbarrier and the others wait
// here for its verdict.
__device__ __forceinline__ bool bar_or(uint32_t id, uint32_t n, bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 q, %1, 0;\n\t"
                 "bar.red.or.pred p, %2, %3, q;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}\n"
                 : "=r"(r)
                 : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
                 : "memory");
    return r != 0;
}

// The softmax barrier of quadrant qd (its two warps).
__device__ __forceinline__ bool softmax_bar_or(uint32_t qd, bool pred)
{
    return bar_or(kBarSoftmax0 + qd, kSmQuadThreads, pred);
}

__device__ __forceinline__ void softmax_bar(uint32_t qd)
{
    asm volatile("bar.sync %0, %1;" ::"r"(kBarSoftmax0 + qd), "r"(kSmQuadThreads) : "memory");
}

// One thread of a role (`leader`) waits on the mbarrier; the role's `n` threads learn the
// outcome at named barrier `id`.  true = the phase completed; false = every thread gives up.
__device__ __forceinline__ bool role_wait(uint64_t *bar, uint32_t parity, int32_t *abort_flag,
                                          bool leader, uint32_t id, uint32_t n)
{
    bool ok = true;
    if (leader)
        ok = wait_bar_c(bar, parity, abort_flag);
    return !bar_or(id, n, !ok);
}

// A descriptor's start-address field is (address >> 4) in its low 14 bits: a descriptor for
// `base + off` is the descriptor for `base` plus off >> 4 (no carry below 256 KiB).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t off_bytes)
{
    return d + static_cast<uint64_t>(off_bytes >> 4);
}

// One arrival per warp: every lane's prior writes are ordered before lane 0's arrive.
__device__ __forceinline__ void warp_arrive(uint64_t *bar, int lane)
{
    __syncwarp();
    if (lane == 0)
        mbar_arrive(bar);
}

// ---------------- Q: power-of-two row scale and the exact two-part E4M3 split ----------------

// Largest bf16 exponent field among the eight values packed in v.
__device__ __forceinline__ uint32_t max_exp8(const uint4 v)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        m = max(m, max((w[i] >> 7) & 0xFFu, (w[i] >> 23) & 0xFFu));
    return m;
}

// Scale exponent s of a Q row whose largest bf16 exponent field is e: 2^s brings the row's
// largest magnitude into [128, 256), inside the E4M3 range (largest finite 448).  Clamped so
// that 2^s and 2^-s are normal floats.
__device__ __forceinline__ int q_scale_exp(uint32_t e)
{
    return min(max(134 - static_cast<int>(e), -126), 126);
}

__device__ __forceinline__ float exp2i(int s) // 2^s for s in [-126, 127]
{
    return __int_as_float((s + 127) << 23);
}

// Two f32 -> packed E4M3 pair (round to nearest even); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_rn(float lo, float hi)
{
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// Packed E4M3 pair -> its two values as f32 (exact).
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t pair, float &lo, float &hi)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(pair)));
    const __half2 h = *reinterpret_cast<const __half2 *>(&h2);
    lo = __low2float(h);
    hi = __high2float(h);
}

// Eight bf16 values (element 0 in the low half of v.x) times 2^s -> E4M3 parts q1 and q2 with
// q1 + q2 = q 2^s; byte i of each result holds element i.
__device__ __forceinline__ void split_q8(const uint4 v, float scale, uint2 &q1, uint2 &q2)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float x0 = __uint_as_float(w[i] << 16) * scale;
        const float x1 = __uint_as_float(w[i] & 0xFFFF0000u) * scale;
        a[i] = e4m3x2_rn(x0, x1);
        float y0, y1;
        e4m3x2_to_f32(a[i], y0, y1);
        b[i] = e4m3x2_rn(x0 - y0, x1 - y1);
    }
    q1 = make_uint2(a[0] | (a[1] << 16), a[2] | (a[3] << 16));
    q2 = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
}

// Packed fp32 pairs: two independent IEEE single-precision operations per instruction.
__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

// (x0, x1) = (s0, s1) * c2 + m2, elementwise (c2, m2 packed pairs).
__device__ __forceinline__ void fma2(float &x0, float &x1, uint32_t s0, uint32_t s1, uint64_t c2, uint64_t m2)
{
    asm("{\n\t.reg .b64 s2, x2;\n\t"
        "mov.b64 s2, {%2, %3};\n\t"
        "fma.rn.f32x2 x2, s2, %4, %5;\n\t"
        "mov.b64 {%0, %1}, x2;\n\t}"
        : "=f"(x0), "=f"(x1)
        : "r"(s0), "r"(s1), "l"(c2), "l"(m2));
}

// a + (p0, p1), elementwise.
__device__ __forceinline__ uint64_t add2(uint64_t a, float p0, float p1)
{
    uint64_t r;
    asm("{\n\t.reg .b64 p2;\n\t"
        "mov.b64 p2, {%1, %2};\n\t"
        "add.rn.f32x2 %0, %3, p2;\n\t}"
        : "=l"(r)
        : "f"(p0), "f"(p1), "l"(a));
    return r;
}

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// A partial page (the query's own page, keys up to its position): the scores of the keys from
// the nq-th on become -inf, so that the max and P of every page with allowed keys take one
// path without per-key predicates (the log2-domain factor is kept positive, so -inf stays -inf
// and its P is 0).
__device__ __forceinline__ void mask_tail(uint32_t (&sv)[16], int nq)
{
    if (nq > 0 && nq < 16) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
            if (e >= nq)
                sv[e] = 0xFF800000u; // -inf
    }
}

// Largest of this thread's 16 scores of a page (tail masked), -inf when no key is allowed.
// Each thread takes the case of its own nq: a page not selected by the row's query (nq = 0)
// costs nothing.
__device__ __forceinline__ float page_max(const uint32_t (&sv)[16], int nq)
{
    if (nq == 0)
        return -INFINITY;
    const float *v = reinterpret_cast<const float *>(sv);
    float a = max3f(v[0], v[1], v[2]), b = max3f(v[3], v[4], v[5]);
    a = max3f(a, v[6], v[7]);
    b = max3f(b, v[8], v[9]);
    a = max3f(a, v[10], v[11]);
    b = max3f(b, v[12], v[13]);
    a = max3f(a, v[14], v[15]);
    return fmaxf(a, b);
}

// p -> (hi, lo) f16 halves of two packed words: hi = p rounded to f16, lo = p - hi (exact in
// f32, formed by one mixed-precision multiply-add with the f16 operand widened exactly) rounded
// to f16.  For p in [2^-3, 256] the pair carries about 22 significant bits; below, the absolute
// error stays under 2^-25.
__device__ __forceinline__ void split_pair_f16_pos(float p0, float p1, uint32_t &hi2, uint32_t &lo2)
{
    asm("{\n\t.reg .b16 h0, h1, m1;\n\t.reg .f32 d0, d1;\n\t"
        "mov.b16 m1, 0xBC00;\n\t" // -1.0 in f16
        "cvt.rn.f16x2.f32 %0, %3, %2;\n\t"
        "mov.b32 {h0, h1}, %0;\n\t"
        "fma.rn.f32.f16 d0, h0, m1, %2;\n\t"
        "fma.rn.f32.f16 d1, h1, m1, %3;\n\t"
        "cvt.rn.f16x2.f32 %1, d1, d0;\n\t}"
        : "=r"(hi2), "=r"(lo2)
        : "f"(p0), "f"(p1));
}

// 16 lanes x 32 bit, two column halves (the 16x32bx2 shape with a split of 16 columns): lanes
// 0-15 of the warp write 8 columns from the address's column, lanes 16-31 from 16 columns on.
__device__ __forceinline__ void tmem_st_16x32bx2_x8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], 16, {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

// The same shape, 32 columns per half (split of 32 columns).
__device__ __forceinline__ void tmem_ld_16x32bx2_x32s(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
                   "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
                   "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_16x32bx2_x32s(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile("tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                 "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
                 "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
                 "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem] with kind::f16: A is read from TMEM (row r at lane r for M = 128;
// for M = 64 at lane 32 (r / 16) + r % 16; keys 2j and 2j + 1 packed in column j), B from a
// shared-memory descriptor.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Wait for this thread's outstanding tcgen05.ld into two 16-register arrays (both routed through
// the asm, so that no use of them is scheduled before the wait).
__device__ __forceinline__ void tmem_ld_wait2x16(uint32_t (&a)[16], uint32_t (&b)[16])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]),
                   "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]),
                   "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15]), "+r"(b[0]), "+r"(b[1]),
                   "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7]),
                   "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]),
                   "+r"(b[14]), "+r"(b[15])::"memory");
}

// P = 2^(s c + negm) of the 16 keys of one row that this thread read of one page (the first nq
// allowed, the tail masked to -inf, so their P is 0), split into f16 hi + lo parts (keys 2j,
// 2j + 1 in word j).  Returns the keys' sum.  As in page_max, each thread takes the case of its
// own nq.
__device__ __forceinline__ float p_page(const uint32_t (&sv)[16], int nq, float c, float negm,
                                        uint32_t (&hi)[8], uint32_t (&lo)[8])
{
    float sum = 0.f;
    if (nq != 0) { // every key allowed, or the tail masked to -inf
        const uint64_t c2 = pack2(c, c), m2 = pack2(negm, negm);
        uint64_t sum2 = 0; // (0.f, 0.f)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float x0, x1;
            fma2(x0, x1, sv[2 * e], sv[2 * e + 1], c2, m2);
            const float p0 = ex2(x0), p1 = ex2(x1);
            sum2 = add2(sum2, p0, p1);
            split_pair_f16_pos(p0, p1, hi[e], lo[e]);
        }
        sum = __uint_as_float(static_cast<uint32_t>(sum2)) + __uint_as_float(static_cast<uint32_t>(sum2 >> 32));
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            hi[e] = lo[e] = 0u;
    }
    return sum;
}

// The hi/lo parts of one page's 16 keys of one row, written back over the 16 columns this thread
// read them from (as the A operand of O += P V): P_hi in the first 8 columns, P_lo in the last 8
// (for lanes 16-31 of the warp, 16 columns further on, as they were read).
__device__ __forceinline__ void store_p(const uint32_t (&hi)[8], const uint32_t (&lo)[8], uint32_t p_addr)
{
    tmem_st_16x32bx2_x8(p_addr, hi);
    tmem_st_16x32bx2_x8(p_addr + 8, lo);
}

// The softmax role's slow path, taken when some row's scores exceed its running max by more
// than 2^8 (always at a group's first step): the row's four threads agree on its max and, when
// a row's max rises, O[r, :] *= alpha[r] once every product issued so far (those of the steps
// before stp) has completed.  Kept out of line so that the common path of the softmax loop stays
// small in the instruction cache.  Every thread of the role calls it; the state comes back by
// value.
struct SlowOut {
    float m_used, l_part;
    bool ok;
};

__device__ __noinline__ SlowOut softmax_slow_path(WsSmem &sm, int row, int qq, int hw, bool any, float lm,
                                                  float m_used, float l_part, bool first_step,
                                                  uint32_t stp, bool sleader, uint32_t o_addr, uint32_t qd)
{
    sm.qmax[row][qq] = any ? lm : -INFINITY;
    softmax_bar(qd);
    const float M = fmaxf(fmaxf(sm.qmax[row][0], sm.qmax[row][1]), fmaxf(sm.qmax[row][2], sm.qmax[row][3]));
    float alpha = 1.f;
    bool rescale = false;
    if (M > m_used + kRescaleLog2) {
        if (m_used != -INFINITY) {
            alpha = ex2(m_used - M);
            rescale = true;
            l_part *= alpha;
        }
        m_used = M;
    }
    // (at a group's first step no row has a max yet, so none rescales)
    if (!first_step && softmax_bar_or(qd, rescale)) {
        // pvs_done of step stp - 1 covers every product issued before it.  Its phase is
        // unambiguous: S of this step was issued after the products of step stp - 3 had
        // completed, and the products of step stp + 2 cannot have run yet.
        const bool ok = !sleader ||
                        wait_bar(&sm.pvs_done[(stp - 1) % kNS], ((stp - 1) / kNS) & 1u, &sm.abort_flag);
        if (softmax_bar_or(qd, !ok))
            return SlowOut{m_used, l_part, false};
        // O[r, :] *= alpha[r]: the row sits in this warp's lanes, and its four threads take 32
        // head dimensions each (lanes 0-15 dims 64 hw .. 64 hw + 31, lanes 16-31 the next 32).
        tc_fence_after();
        uint32_t o[32];
        tmem_ld_16x32bx2_x32s(o_addr + 64 * hw, o);
        tmem_ld_wait(o);
#pragma unroll
        for (int e = 0; e < 32; ++e)
            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st_16x32bx2_x32s(o_addr + 64 * hw, o);
        tmem_st_wait();
    }
    return SlowOut{m_used, l_part, true};
}

// tmap_k: the K pages as a 2-D byte tensor [n_phys * Hkv * 64 rows][128], boxes of 64 x 128
// with the 128-byte swizzle, so that one copy lands a page as the K-major operand of S.
// kDyn: groups from the launch's work counter (ragged batches) instead of a fixed stride; two
// instantiations, so that each carries the code of one schedule only.
template <bool kDyn>
__global__ void __launch_bounds__(kThreads, 1)
    k_union_attn_ws(const AttnLaunch L, const __grid_constant__ CUtensorMap tmap_k)
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
        // Arrivals from the decode and softmax roles are one per warp (after __syncwarp).
        for (int s = 0; s < kNJ; ++s) {
            mbar_init(&sm.job_full[s], 1);
            mbar_init(&sm.job_empty[s], kDecThreads / 32 + 2 + kSmThreads / 32 + kEpiThreads / 32);
        }
        mbar_init(&sm.qraw_full, 1);
        mbar_init(&sm.qraw_empty, kEpiThreads / 32);
        for (int s = 0; s < kNKP; ++s)
            mbar_init(&sm.kst_full[s], 1);
        for (int s = 0; s < kNSV; ++s) {
            mbar_init(&sm.vst_full[s], 1);
            mbar_init(&sm.vst_empty[s], kDecThreads / 32);
        }
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&sm.s_done[s], 1);
            mbar_init(&sm.pvs_done[s], 1);
            mbar_init(&sm.pv_ready[s], kSmThreads / 32 + kDecThreads / 32);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.q_full[s], kEpiThreads / 32);
            mbar_init(&sm.q_empty[s], 1);
            mbar_init(&sm.l_full[s], kSmThreads / 32);
            mbar_init(&sm.o_free[s], kEpiThreads / 32);
        }
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.drain_bar, 2); // one commit from each MMA-issuing warp
        sm.abort_flag = 0;
        sm.k_issued = 0;
        sm.v_issued = 0;
        sm.q_issued = 0;
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

    if (warp == kWarpLoad) {
        // ---------------- load: group records, Q rows, union pages -> stages ----------------
        // Works one group ahead: while it issues the pages of group n it has already published
        // the record of group n + 1, and it copies group n + 1's Q rows as soon as the raw Q
        // buffer is free (the epilogue warps then prepare that Q tile in the middle of group n).
        // The latency of its dependent global loads (group -> query IDs -> positions and
        // membership words) stays off the other roles' path.  Every lane polls its mbarriers;
        // lane 0 issues the copies.
        auto lwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(kFull, wait_bar_c(bar, parity, &sm.abort_flag));
        };
        struct GMeta {
            int b, h, gsz, R, u0, nU, pg0, pg1, pg2, pg3;
            int32_t tok_l, cu_b;   // lane l: query l of the group
            uint32_t w0_l, w1_l;   // lane l: its membership words of the first two union pages
        };
        // The next group with union pages; groups without any get their zero rows.  With
        // kDyn (a ragged batch) groups come from the launch's work counter: ticket t is
        // group n_groups - 1 - t, so the longest sequences' groups, which carry the largest
        // unions, start first and short groups fill the end, and every CTA stays busy until
        // the last tickets are gone (lane 0 holds the next ticket, taken one group early so
        // that the atomic's round trip overlaps the current group's copies; a CTA never holds
        // more than one unused ticket, and once one is past the last group so are all later
        // ones).  Otherwise CTA i takes groups i, i + gridDim.x, ...: on a single sequence this
        // measured faster than the counter.  A record that would address outside the launch's
        // buffers (sequence, head, size or a member token out of range) is skipped and
        // recorded as PW_ERR_INVALID_ARG.
        int ticket = kDyn && lane == 0 ? atomicAdd(L.sched, 1) : 0;
        int64_t g_static = blockIdx.x;
        auto next_index = [&]() -> int64_t {
            if (!kDyn) {
                const int64_t gi = g_static;
                g_static += gridDim.x;
                return gi < L.n_groups ? gi : -1;
            }
            const int t = __shfl_sync(kFull, ticket, 0);
            if (t >= L.n_groups)
                return -1;
            if (lane == 0)
                ticket = atomicAdd(L.sched, 1);
            return L.n_groups - 1 - t;
        };
        auto next_group = [&](GMeta &m) -> bool {
            for (;;) {
                const int64_t gi = next_index();
                if (gi < 0)
                    return false;
                const int b = L.gmeta[3 * gi], h = L.gmeta[3 * gi + 1];
                const int gsz = L.gsize[gi], R = gsz * L.G;
                const int u0 = L.union_off[gi], nU = L.union_off[gi + 1] - u0;
                if (!group_scalars_ok(L, b, h, gsz, nU))
                    continue;
                const int32_t cu_b = L.cu[b], cu_e = L.cu[b + 1];
                const int32_t tok_l = lane < gsz ? L.qids[gi * L.g + lane] : cu_b;
                if (!__all_sync(kFull, tok_l >= cu_b && tok_l < cu_e)) {
                    if (lane == 0)
                        set_status(L.status, PW_ERR_INVALID_ARG);
                    continue;
                }
                if (nU == 0) {
                    for (int idx = lane; idx < R * 16; idx += 32) {
                        const int r = idx >> 4, c = idx & 15, mi = r / L.G;
                        const int64_t tok = L.qids[gi * L.g + mi];
                        const int hq = h * L.G + (r - mi * L.G);
                        reinterpret_cast<uint4 *>(L.O + (static_cast<size_t>(tok) * L.Hq + hq) * kHeadDim)[c] =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    continue;
                }
                m.b = b;
                m.h = h;
                m.gsz = gsz;
                m.R = R;
                m.u0 = u0;
                m.nU = nU;
                m.tok_l = lane < gsz ? tok_l : 0;
                m.cu_b = cu_b;
                m.pg0 = L.union_pages[u0];
                m.pg1 = nU > 1 ? L.union_pages[u0 + 1] : m.pg0;
                m.pg2 = nU > 2 ? L.union_pages[u0 + 2] : m.pg0;
                m.pg3 = nU > 3 ? L.union_pages[u0 + 3] : m.pg0;
                const uint32_t *bitrow = L.bits + (static_cast<size_t>(m.tok_l) * L.Hkv + h) * L.words;
                m.w0_l = lane < gsz ? __ldg(bitrow + page_word(L, m.pg0)) : 0u;
                m.w1_l = lane < gsz ? __ldg(bitrow + page_word(L, m.pg1)) : 0u;
                return true;
            }
        };
        // Record of job n (or the end marker when m is null) into its ring slot.
        auto publish = [&](uint32_t n, const GMeta *m) -> bool {
            const uint32_t jb = n % kNJ;
            if (!lwait(&sm.job_empty[jb], ((n / kNJ) & 1u) ^ 1u))
                return false;
            GroupJob &J = sm.job[jb];
            if (m != nullptr) {
#pragma unroll
                for (int r0 = 0; r0 < 64; r0 += 32) {
                    const int r = r0 + lane;
                    const int mi = min(r / L.G, 31);
                    const int32_t t = __shfl_sync(kFull, m->tok_l, mi);
                    J.tok[r] = r < m->R ? t : 0;
                    J.pos[r] = r < m->R ? t - m->cu_b : 0;
                }
                J.word0[0][lane] = m->w0_l;
                J.word0[1][lane] = m->w1_l;
            }
            if (lane == 0) {
                J.nU = m != nullptr ? m->nU : -1;
                if (m != nullptr) {
                    J.b = m->b;
                    J.h = m->h;
                    J.R = m->R;
                    J.u0 = m->u0;
                    J.pg0 = m->pg0;
                    J.pg1 = m->pg1;
                    J.pg2 = m->pg2;
                    J.pg3 = m->pg3;
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.job_full[jb]);
            return true;
        };
        // Q rows of job n: query qi's G heads are G consecutive rows of Q.  The raw buffer is
        // free (the caller waited for it).
        auto copy_q = [&](uint32_t n, const GMeta &m) {
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.qraw_full, static_cast<uint32_t>(m.R) * 256u);
                sm.q_issued = n + 1;
            }
            __syncwarp();
            if (lane < m.gsz)
                bulk_g2s(sm.q_raw + lane * L.G * 256,
                         L.Q + (static_cast<size_t>(m.tok_l) * L.Hq + m.h * L.G) * kHeadDim,
                         static_cast<uint32_t>(L.G) * 256u, &sm.qraw_full);
        };
        uint32_t it = 0, stp = 0;
        bool stop = false, has_cur = false;
        GMeta cur{}, nxt{};
        // Iteration n publishes job n (the next group's record, or the end marker), then issues
        // the pages of job n - 1 and, as soon as the raw Q buffer is free, job n's Q rows.  One
        // call site for each keeps this role's code small.
        for (uint32_t n = 0; !stop; ++n) {
            const bool has_nxt = next_group(nxt);
            if (!publish(n, has_nxt ? &nxt : nullptr)) {
                stop = true;
                break;
            }
            bool q_pending = has_nxt; // Q rows of job n, once job n - 1's raw rows are used
            // phase n - 1 of qraw_empty (released by job n - 1's split; for n = 0 the phase
            // before the first, which reads as complete)
            const uint32_t q_parity = (n & 1u) ^ 1u;
            const int b = cur.b, h = cur.h, u0 = cur.u0, nU = has_cur ? cur.nU : 0;
            for (int j0 = 0; j0 < nU && !stop; j0 += 32) {
                const int phys = j0 + lane < nU ? phys_page(L, b, L.union_pages[u0 + j0 + lane]) : 0;
                const int cnt = min(32, nU - j0); // j0 is even: a step never straddles chunks
                for (int jj = 0; jj < cnt && !stop; jj += 2, ++stp) {
                    const int np = min(2, cnt - jj);
                    const int32_t row0 = (__shfl_sync(kFull, phys, jj) * L.Hkv + h) * 64;
                    const int32_t row1 = (__shfl_sync(kFull, phys, min(jj + 1, 31)) * L.Hkv + h) * 64;
                    // K: both pages of the step into one stage pair, on one barrier
                    // the pair is free once S of step stp - 3 has completed
                    const uint32_t kp = stp % kNKP;
                    if (!lwait(&sm.s_done[kp], ((stp / kNKP) & 1u) ^ 1u)) {
                        stop = true;
                        break;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&sm.kst_full[kp], static_cast<uint32_t>(np) * kPageBytes);
                        tma_load_2d(sm.stage_k[kp][0], &tmap_k, 0, row0, &sm.kst_full[kp]);
                        if (np == 2)
                            tma_load_2d(sm.stage_k[kp][1], &tmap_k, 0, row1, &sm.kst_full[kp]);
                        sm.k_issued = stp + 1;
                    }
                    // V: page by page
                    for (int k = 0; k < np; ++k, ++it) {
                        const uint32_t vs = it % kNSV;
                        if (!lwait(&sm.vst_empty[vs], ((it / kNSV) & 1u) ^ 1u)) {
                            stop = true;
                            break;
                        }
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&sm.vst_full[vs], kPageBytes);
                            bulk_g2s(sm.stage_v[vs], L.V + static_cast<size_t>(k == 0 ? row0 : row1) * 128,
                                     kPageBytes, &sm.vst_full[vs]);
                            sm.v_issued = it + 1;
                        }
                    }
                    __syncwarp();
                    // the next job's Q rows, as soon as the raw buffer is free (no wait here)
                    if (!stop && q_pending && __all_sync(kFull, mbar_try_wait(&sm.qraw_empty, q_parity))) {
                        copy_q(n, nxt);
                        q_pending = false;
                    }
                }
            }
            if (!stop && q_pending) {
                if (!lwait(&sm.qraw_empty, q_parity)) {
                    stop = true;
                    break;
                }
                copy_q(n, nxt);
            }
            if (!has_nxt)
                break;
            cur = nxt;
            has_cur = true;
        }
    } else if (warp == kWarpMma || warp == kWarpPv) {
        // ---------------- MMA issue: two warps ----------------
        // Warp kWarpMma issues S of every step, as soon as its K pair has landed and the products
        // of the step three before (which read its S/P buffer as P) are complete, so it runs up
        // to three steps ahead; warp kWarpPv issues O += P V of every step once its P is written
        // and its V tiles decoded.  Each warp runs its loop in lockstep: every lane polls the
        // mbarriers and a vote makes each decision warp-uniform; the elected lane (always lane
        // 0) issues the tensor-core instructions and the commits, which track that lane's MMAs.
        auto wwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            const bool ok = wait_bar(bar, parity, &sm.abort_flag); // every lane polls
            return __all_sync(kFull, ok);
        };
        const bool is_s = warp == kWarpMma;
        const uint64_t dsw = sdesc_sw128(0u, 16, 1024);    // K-major, address added below
        const uint64_t dmn = sdesc_sw128(0u, 8192, 1024);  // V, MN-major (dims contiguous)
        constexpr uint32_t idesc_pv = idesc_f16_f32(64, 128, false, true);
        uint32_t stp = 0;
        bool ok = true;
        for (uint32_t nact = 0; ok; ++nact) {
            const uint32_t jb = nact % kNJ;
            if (!wwait(&sm.job_full[jb], (nact / kNJ) & 1u))
                break;
            const int nU = sm.job[jb].nU;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.job_empty[jb]);
            if (nU < 0)
                break;
            const uint32_t qb = nact & 1u;
            uint64_t aq1 = 0, aq2 = 0;
            if (is_s) {
                if (!wwait(&sm.q_full[qb], (nact >> 1) & 1u))
                    break;
                aq1 = desc_add(dsw, smem_u32(sm.q[qb][0]));
                aq2 = desc_add(dsw, smem_u32(sm.q[qb][1]));
            }
            for (int s0 = 0; s0 < nU; s0 += 2, ++stp) {
                const uint32_t np = static_cast<uint32_t>(min(2, nU - s0));
                const bool last = s0 + static_cast<int>(np) == nU;
                const uint32_t sb = stp % kNS; // S/P buffer (and K stage pair) of the step
                if (is_s) {
                    // S buffer sb holds the P of step stp - 3: S may overwrite it once the
                    // products of that step have read it.
                    if (!wwait(&sm.kst_full[sb], (stp / kNS) & 1u) ||
                        (stp >= kNS && !wwait(&sm.pvs_done[sb], ((stp / kNS) & 1u) ^ 1u))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bk = desc_add(dsw, smem_u32(sm.stage_k[sb][0]));
                    const uint32_t ds = tmem + kColS * sb;
                    const uint32_t idesc_s = idesc_e4m3_f32(64, static_cast<int>(64 * np));
                    if (elect_one()) {
                        // S' = q1 K^T + q2 K^T: four k-steps of 32 dims for each part
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f8_ss(ds, aq1 + 2u * kk, bk + 2u * kk, idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f8_ss(ds, aq2 + 2u * kk, bk + 2u * kk, idesc_s, 1u);
                        mma_commit(&sm.s_done[sb]);
                        if (last)
                            mma_commit(&sm.q_empty[qb]);
                    }
                    __syncwarp();
                } else {
                    // P of the step in S/P buffer sb, its V tiles in step slot stp % 2; the first
                    // products of group g overwrite O, so the epilogue must have read group
                    // g - 1's.
                    const uint32_t vsl = stp & 1u;
                    if (!wwait(&sm.pv_ready[sb], (stp / kNS) & 1u) ||
                        (s0 == 0 && nact > 0 && !wwait(&sm.o_free[(nact - 1) & 1u], ((nact - 1) >> 1) & 1u))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // O += P V, P read from TMEM where the softmax wrote it (the step's S buffer),
                    // V (K = keys, N = dims) from its MN-major f16 tile.
                    const uint32_t d = tmem + kColO;
                    const uint32_t pa = tmem + kColS * sb;
                    const uint64_t bd0 = desc_add(dmn, smem_u32(&sm.v[vsl][0][0][0]));
                    if (elect_one()) {
                        for (uint32_t k = 0; k < np; ++k) {
                            const uint64_t bd = bd0 + ((k * sizeof(sm.v[0][0])) >> 4); // page k's tile
                            const bool first = s0 == 0 && k == 0;
                            // keys 16 kk .. 16 kk + 15: P_hi in columns 16 kk .. 16 kk + 7 of the
                            // page, P_lo in the next 8
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint32_t a = pa + 64 * k + 16 * kk;
                                mma_f16_ts(d, a, bd + 128u * kk, idesc_pv, (first && kk == 0) ? 0u : 1u);
                                mma_f16_ts(d, a + 8, bd + 128u * kk, idesc_pv, 1u);
                            }
                        }
                        mma_commit(&sm.pvs_done[sb]);
                        if (last)
                            mma_commit(&sm.o_full);
                    }
                    __syncwarp();
                }
            }
        }
    } else if (warp < kWarpSm0) {
        // ---------------- decode: E4M3 -> f16 V tiles, one step (one or two pages) at a time ----
        // Each warp waits on the mbarriers itself (every lane polls, a vote decides), so the four
        // warps never wait for one another.  The tiles of step n go to step slot n % 2, free again
        // once the products of step n - 2 are complete.
        auto dwait = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(kFull, wait_bar_c(bar, parity, &sm.abort_flag));
        };
        uint32_t it = 0, stp = 0, nact = 0;
        bool ok = true;
        for (;;) {
            const uint32_t jb = nact % kNJ;
            if (!dwait(&sm.job_full[jb], (nact / kNJ) & 1u)) {
                ok = false;
                break;
            }
            const int nU = sm.job[jb].nU;
            warp_arrive(&sm.job_empty[jb], lane);
            if (nU < 0)
                break;
            for (int s0 = 0; s0 < nU; s0 += 2, ++stp) {
                const int np = min(2, nU - s0);
                // V step slot sb was last read by the products of step stp - 2.  Their phase of
                // pvs_done is unambiguous: this warp waited for those of step stp - 5 before
                // decoding step stp - 3, and the products of step stp + 1 need tiles not yet made.
                const uint32_t sb = stp & 1u, st0 = it % kNSV, st1 = (it + 1) % kNSV;
                if (!((stp < 2 || dwait(&sm.pvs_done[(stp - 2) % kNS], ((stp - 2) / kNS) & 1u)) &&
                      dwait(&sm.vst_full[st0], (it / kNSV) & 1u) &&
                      (np < 2 || dwait(&sm.vst_full[st1], ((it + 1) / kNSV) & 1u)))) {
                    ok = false;
                    break;
                }
#pragma unroll 1
                for (int k = 0; k < np; ++k)
                    decode_page_f16<kDecThreads>(sm.stage_v[k == 0 ? st0 : st1], sm.v[sb][k], tid);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&sm.pv_ready[stp % kNS]);
                    mbar_arrive(&sm.vst_empty[st0]);
                    if (np == 2)
                        mbar_arrive(&sm.vst_empty[st1]);
                }
                it += np;
            }
            if (!ok)
                break;
            ++nact;
        }
    } else if (warp < kWarpEpi0) {
        // ---------------- softmax (256 threads) ----------------
        // Four threads share a row: warp (quadrant qd, half hw) reads TMEM lanes of rows
        // 16 qd .. 16 qd + 15 and, of each page, keys 32 hw .. 32 hw + 31; lane / 16 picks 16 of
        // those keys.  A step is one or two pages.  A row's running max m is identical in its
        // four threads and changes only on the slow path, which runs when some element of some
        // row exceeds its m by more than 2^8 (one OR over all 256 threads decides), so the
        // common path needs no exchange.
        const int sw = warp - kWarpSm0;     // 0..7
        const bool sleader = sw < 4 && lane == 0; // the quadrant's one mbarrier waiter
        const int qd = sw & 3;              // TMEM lane quadrant
        const int hw = sw >> 2;             // key half of each page read by this warp
        const int row = 16 * qd + (lane & 15);
        const int qq = 2 * hw + (lane >> 4); // 16-key quarter of each page owned by this thread
        // |log2-domain factor|: when the factor is negative, the Q tile is negated instead
        const float acrow = fabsf(L.sm_scale * L.k_scale * kLog2e);
        const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
        uint32_t stp = 0, nact = 0;
        auto allowed = [&](int pg, uint32_t word, int pos, int own) -> int { // keys of page pg in my quarter
            int n_allow = 0;
            if ((word >> (pg & 31)) & 1u)
                n_allow = pg < own ? 64 : (pg == own ? (pos & 63) + 1 : 0);
            return min(max(n_allow - 16 * qq, 0), 16);
        };
        bool ok = true;
        for (;;) {
            // the group record; its Q scale exponents are written with the Q tile
            const uint32_t jb = nact % kNJ;
            bool got = true;
            if (sleader) {
                got = wait_bar_c(&sm.job_full[jb], (nact / kNJ) & 1u, &sm.abort_flag);
                if (got && sm.job[jb].nU >= 0)
                    got = wait_bar_c(&sm.q_full[nact & 1u], (nact >> 1) & 1u, &sm.abort_flag);
            }
            if (softmax_bar_or(qd, !got)) {
                ok = false;
                break;
            }
            const GroupJob &J = sm.job[jb];
            const int nU = J.nU;
            if (nU < 0)
                break;
            const int h = J.h, R = J.R, u0 = J.u0;
            const bool valid = row < R;
            const int32_t tok = J.tok[row];
            const int pos = J.pos[row], own = pos >> 6;
            const uint32_t *bitrow = L.bits + (static_cast<size_t>(tok) * L.Hkv + h) * L.words;
            // S arrives scaled by 2^s (the row's Q scale): fold 2^-s into the log2-domain factor
            const float inv = exp2i(-J.qexp[row]);
            // (floored at a tiny positive value, so that a masked key's -inf score never meets a
            // zero factor; a zero factor makes all allowed keys equal either way)
            const float c_r = fmaxf(acrow * inv, 1e-30f);
            // Union page ids and my membership words, software-pipelined so that no step waits
            // on a global load: at the top of each step the words of the next step's pages and
            // the ids of the pages two steps ahead are requested; at its end, when they have
            // landed, they move down one stage.
            int pgA = J.pg0, pgB = J.pg1;     // this step
            uint32_t wA = valid ? J.word0[0][row / L.G] : 0u;
            uint32_t wB = valid ? J.word0[1][row / L.G] : 0u;
            int pn0 = J.pg2, pn1 = J.pg3;     // next step (ids known)
            uint32_t wn0 = 0u, wn1 = 0u;      // next step (words requested at the top of this one)
            int pnn0 = pn0, pnn1 = pn1;       // two steps ahead (ids requested at the top of this one)
            warp_arrive(&sm.job_empty[jb], lane);
            const uint32_t ob = nact & 1u; // lsum buffer of the group
            const uint32_t o_addr = tmem + lane_base + kColO;
            float m_used = -INFINITY, l_part = 0.f;
            for (int s0 = 0; s0 < nU; s0 += 2, ++stp) {
                const int np = min(2, nU - s0);
                if (s0 + 2 < nU && valid)
                    wn0 = __ldg(bitrow + page_word(L, pn0));
                if (s0 + 3 < nU && valid)
                    wn1 = __ldg(bitrow + page_word(L, pn1));
                if (s0 + 4 < nU)
                    pnn0 = L.union_pages[u0 + s0 + 4];
                if (s0 + 5 < nU)
                    pnn1 = L.union_pages[u0 + s0 + 5];
                const uint32_t sb = stp % kNS;
                // Every warp waits for S itself (all lanes poll, the warp decides by vote), so the
                // warps are not lined up at a barrier here.  Every abort decision of this role is
                // still collective (a thread that left alone would strand the others at the named
                // barrier or in a warp-wide TMEM load): a warp whose wait gave up carries that to
                // the vote below.
                // The scores of both pages of the step arrive in one round trip and stay in
                // registers for the max and for P.  For a one-page step the second page's
                // columns hold stale values; they are all masked.
                const bool s_ok = __all_sync(kFull, wait_bar(&sm.s_done[sb], (stp / kNS) & 1u, &sm.abort_flag));
                tc_fence_after();
                const uint32_t s_addr = tmem + lane_base + kColS * sb + 32 * hw;
                uint32_t sa[16], sc[16];
                tmem_ld_16x32bx2_x16(s_addr, sa);
                tmem_ld_16x32bx2_x16(s_addr + 64, sc);
                const int nqA = allowed(pgA, wA, pos, own);
                const int nqB = np == 2 ? allowed(pgB, wB, pos, own) : 0;
                tmem_ld_wait2x16(sa, sc);
                mask_tail(sa, nqA);
                mask_tail(sc, nqB);
                float lm = fmaxf(page_max(sa, nqA), page_max(sc, nqB));
                const bool any = nqA > 0 || nqB > 0;
                if (any)
                    lm *= c_r;
                if (softmax_bar_or(qd, !s_ok || (any && lm > m_used + kRescaleLog2))) {
                    if (softmax_bar_or(qd, !s_ok)) {
                        ok = false;
                        break;
                    }
                    const SlowOut so = softmax_slow_path(sm, row, qq, hw, any, lm, m_used, l_part, s0 == 0,
                                                         stp, sleader, o_addr, qd);
                    m_used = so.m_used;
                    l_part = so.l_part;
                    if (!so.ok) {
                        ok = false;
                        break;
                    }
                    // The scores again (still in TMEM): keeping them in registers across the
                    // out-of-line call would spill them.
                    tmem_ld_16x32bx2_x16(s_addr, sa);
                    tmem_ld_16x32bx2_x16(s_addr + 64, sc);
                    tmem_ld_wait2x16(sa, sc);
                    mask_tail(sa, nqA);
                    mask_tail(sc, nqB);
                }
                const float negm = m_used == -INFINITY ? 0.f : -m_used;
                // P of each page goes back over that page's S columns, where the products read it
                // as their A operand; the products of step stp - 3, which read these columns as P,
                // completed before S of this step was issued.
                // One call site for both pages (page 1's scores move into sa after page 0).
#pragma unroll 1
                for (int k = 0; k < np; ++k) {
                    uint32_t hi[8], lo[8];
                    l_part += p_page(sa, k == 0 ? nqA : nqB, c_r, negm, hi, lo);
                    store_p(hi, lo, s_addr + 64 * k);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        sa[e] = sc[e];
                }
                tmem_st_wait();
                tc_fence_before();
                warp_arrive(&sm.pv_ready[sb], lane);

                pgA = pn0;
                pgB = pn1;
                wA = wn0;
                wB = wn1;
                pn0 = pnn0;
                pn1 = pnn1;
            }
            if (!ok)
                break;
            // Publish the row-sum partials of this group for the epilogue warps.  lsum[ob] was
            // last read by the epilogue of group nact - 2, which released it with o_free[ob].
            // (The phase is unambiguous: S of this group's steps implies the products of group
            // nact - 3, and so the epilogue's read of group nact - 4, are complete.)
            ok = !sleader || wait_bar_c(&sm.o_free[ob], ((nact >> 1) & 1u) ^ 1u, &sm.abort_flag);
            if (softmax_bar_or(qd, !ok)) {
                ok = false;
                break;
            }
            sm.lsum[ob][row][qq] = l_part;
            warp_arrive(&sm.l_full[ob], lane);
            ++nact;
        }
    } else {
        // ---------------- epilogue (128 threads): Q tiles, and O of finished groups ----------------
        // Per group n: first the Q tile of group n + 1 (its raw rows land while group n runs; the
        // split into two E4M3 parts is off every other role's path here), then the output of
        // group n once its last product is done.
        // Output: warp e reads TMEM lane quadrant e, so thread (e, lane) holds head dimension
        // 32 e + lane of every row and each row's 32 dimensions leave as one 64-byte store per
        // warp.  Row metadata (output row index, 1 / l) is computed lane-parallel, 32 rows at a
        // time, and broadcast with shuffles.  One thread waits on each mbarrier; the others
        // learn the outcome at named barrier kBarEpilogue.
        const int eq = warp - kWarpEpi0;
        const int et = tid - kWarpEpi0 * 32; // 0..127
        const bool eleader = et == 0;
        const uint32_t lane_base = static_cast<uint32_t>(32 * eq) << 16;
        // The softmax works with |log2-domain factor|; a negative factor's sign goes into Q.
        const float qsign = L.sm_scale * L.k_scale < 0.f ? -1.f : 1.f;
        // Q tile of group m: scaled, split into two E4M3 parts, written to buffer m % 2.
        // Returns false when a wait gave up; nU_out < 0 marks the end.
        auto prep_q = [&](uint32_t m, int &nU_out) -> bool {
            const uint32_t jb = m % kNJ, qb = m & 1u;
            if (!role_wait(&sm.job_full[jb], (m / kNJ) & 1u, &sm.abort_flag, eleader, kBarEpilogue,
                           kEpiThreads))
                return false;
            GroupJob &J = sm.job[jb];
            const int R = J.R;
            nU_out = J.nU;
            if (nU_out < 0)
                return true;
            // Q tile buffer qb was last read by the last S of group m - 2; the raw rows of
            // group m have landed.
            bool got = true;
            if (eleader)
                got = wait_bar_c(&sm.q_empty[qb], ((m >> 1) & 1u) ^ 1u, &sm.abort_flag) &&
                      wait_bar_c(&sm.qraw_full, m & 1u, &sm.abort_flag);
            if (bar_or(kBarEpilogue, kEpiThreads, !got))
                return false;
            // Row r of the tile is query head h G + r % G of query r / G.  Sixteen consecutive
            // lanes hold one row (eight dims each) and agree on its scale.  The loop stays rolled:
            // this path has time to spare, and its unrolled code crowded the instruction cache
            // that the softmax loop runs from.
#pragma unroll 1
            for (int rep = 0; rep < 1024 / kEpiThreads; ++rep) {
                const int qn = et + kEpiThreads * rep;
                const int row = qn >> 4, c = qn & 15;
                const uint4 val = row < R ? *reinterpret_cast<const uint4 *>(sm.q_raw + row * 256 + c * 16)
                                          : make_uint4(0u, 0u, 0u, 0u);
                uint32_t e = max_exp8(val);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1)
                    e = max(e, __shfl_xor_sync(kFull, e, o));
                const int sexp = q_scale_exp(e);
                uint2 q1, q2;
                split_q8(val, qsign * exp2i(sexp), q1, q2);
                const uint32_t off = swz(row, c >> 1) + 8u * (c & 1);
                *reinterpret_cast<uint2 *>(sm.q[qb][0] + off) = q1;
                *reinterpret_cast<uint2 *>(sm.q[qb][1] + off) = q2;
                if (c == 0)
                    J.qexp[row] = sexp;
            }
            fence_proxy_async_smem();
            warp_arrive(&sm.q_full[qb], lane);
            warp_arrive(&sm.qraw_empty, lane);
            return true;
        };
        // Iteration m prepares the Q tile of job m, then outputs group m - 1; one call site for
        // each keeps this role's code small.
        bool prev = false; // group m - 1 exists
        for (uint32_t m = 0;; ++m) {
            int nU_m = -1;
            if (!prep_q(m, nU_m))
                break;
            if (!prev) {
                if (nU_m < 0)
                    break;
                prev = true;
                continue;
            }
            // output of group n = m - 1
            const uint32_t n = m - 1;
            const uint32_t jb = n % kNJ, ob = n & 1u; // lsum buffer of the group
            const GroupJob &J = sm.job[jb];
            const int h = J.h, R = J.R;
            bool got = true;
            if (eleader)
                got = wait_bar_lazy(&sm.o_full, n & 1u, &sm.abort_flag) &&
                      wait_bar_lazy(&sm.l_full[ob], (n >> 1) & 1u, &sm.abort_flag);
            if (bar_or(kBarEpilogue, kEpiThreads, !got))
                break;
            // O in TMEM: row r at lane 32 (r / 16) + r % 16 of quadrant r / 16, head dimensions
            // along the columns.  Warp eq takes rows 16 eq .. 16 eq + 15; lanes 0-15 and 16-31
            // take 32 dimensions each per load, so each thread writes 64 contiguous bytes of a row.
            tc_fence_after();
            const uint32_t o_addr = tmem + lane_base + kColO;
            const int r = 16 * eq + (lane & 15), half = lane >> 4;
            float inv = 0.f;
            uint16_t *orow = nullptr;
            if (r < R) {
                const int mi = r / L.G;
                orow = L.O + static_cast<size_t>(J.tok[r] * L.Hq + h * L.G + (r - mi * L.G)) * kHeadDim;
                const float l_row = sm.lsum[ob][r][0] + sm.lsum[ob][r][1] + sm.lsum[ob][r][2] + sm.lsum[ob][r][3];
                inv = l_row > 0.f ? L.v_scale / l_row : 0.f;
            }
#pragma unroll 1
            for (int cb = 0; cb < kHeadDim; cb += 64) {
                uint32_t o[32];
                tmem_ld_16x32bx2_x32s(o_addr + cb, o);
                tmem_ld_wait(o);
                if (r < R) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                                        __uint_as_float(o[2 * e + 1]) * inv);
                        pk[e] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + cb + 32 * half);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            tc_fence_before();
            warp_arrive(&sm.o_free[ob], lane);
            warp_arrive(&sm.job_empty[jb], lane);
            if (nU_m < 0)
                break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (sm.abort_flag != 0) {
        set_status(L.status, PW_ERR_TIMEOUT);
        // Let copies and products still in flight land before the CTA exits (bounded waits):
        // the last copy issued on each stage, and every product issued so far.
        if (tid == 0) {
            const uint32_t nk = sm.k_issued, nv = sm.v_issued;
            for (uint32_t s = 0; s < kNKP && s < nk; ++s) {
                const uint32_t last = s + ((nk - 1 - s) / kNKP) * kNKP;
                (void)mbar_wait(&sm.kst_full[s], (last / kNKP) & 1u);
            }
            for (uint32_t s = 0; s < kNSV && s < nv; ++s) {
                const uint32_t last = s + ((nv - 1 - s) / kNSV) * kNSV;
                (void)mbar_wait(&sm.vst_full[s], (last / kNSV) & 1u);
            }
            if (sm.q_issued > 0)
                (void)mbar_wait(&sm.qraw_full, (sm.q_issued - 1) & 1u);
        }
        if (warp == kWarpMma || warp == kWarpPv) { // each commit covers its own warp's MMAs
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

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no link to libcuda).
EncodeTiledFn encode_tiled()
{
    static const EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

} // namespace

cudaError_t attn_ws_launch(const AttnLaunch &L, cudaStream_t st)
{
    if (L.n_groups == 0)
        return cudaSuccess;
    // Page rows are addressed with 32-bit tensor coordinates.
    const uint64_t k_rows = static_cast<uint64_t>(L.n_phys) * L.Hkv * 64;
    if (L.n_phys < 1 || k_rows > 0x7FFFFFFFull)
        return cudaErrorInvalidValue;
    const EncodeTiledFn enc = encode_tiled();
    if (enc == nullptr)
        return cudaErrorNotSupported;
    CUtensorMap tmap_k;
    const cuuint64_t dims[2] = {128, k_rows};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, 64};
    const cuuint32_t estrides[2] = {1, 1};
    if (enc(&tmap_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(L.K), dims, strides,
            box, estrides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const size_t smem = sizeof(WsSmem) + 1024;
    auto kern = L.dyn_sched ? k_union_attn_ws<true> : k_union_attn_ws<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    const int64_t grid = L.n_groups < sms ? L.n_groups : sms;
    if (L.dyn_sched && (e = cudaMemsetAsync(L.sched, 0, sizeof(int32_t), st)) != cudaSuccess)
        return e;
    kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(L, tmap_k);
    return cudaGetLastError();
}

} // namespace pw
