// pw_attn_common.cuh -- device helpers shared by the union-attention kernels: operand-tile
// swizzle, exact E4M3 -> bf16 (integer bit operations) and E4M3 -> f16 (hardware cvt) decodes,
// the bf16 and f16 hi/lo splits of P.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "pw_internal.h"
#include "pw_sm100.cuh"

namespace pw {
namespace attn {

constexpr int kPageBytes = 64 * 128; // one kv head's page, E4M3
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;

// Physical slot of logical page pg of sequence b through the page table.  A page outside the
// table's row (a table narrower than the sequence) or a slot outside [0, n_phys) records
// PW_ERR_INVALID_ARG and gives slot 0, so that nothing is read outside the caller's buffers.
__device__ __forceinline__ int phys_page(const AttnLaunch &L, int b, int pg)
{
    if (pg < 0 || pg >= L.max_pages) {
        set_status(L.status, PW_ERR_INVALID_ARG);
        return 0;
    }
    const int phys = L.page_table[static_cast<size_t>(b) * L.max_pages + pg];
    if (phys < 0 || phys >= L.n_phys) {
        set_status(L.status, PW_ERR_INVALID_ARG);
        return 0;
    }
    return phys;
}

// Word of a membership bitset row holding page pg's bit, kept inside the row for any pg.
__device__ __forceinline__ uint32_t page_word(const AttnLaunch &L, int pg)
{
    const uint32_t w = static_cast<uint32_t>(pg) >> 5;
    return w < static_cast<uint32_t>(L.words) ? w : static_cast<uint32_t>(L.words - 1);
}

// Whether the scalars of group gi's record address only what the launch owns: sequence and kv
// head in range, 1..g members and a non-negative union length.  (The member tokens are checked
// against the sequence by the caller.)  A bad record is recorded as PW_ERR_INVALID_ARG.
__device__ __forceinline__ bool group_scalars_ok(const AttnLaunch &L, int b, int h, int gsz, int nU)
{
    const bool ok = b >= 0 && b < L.B && h >= 0 && h < L.Hkv && gsz >= 1 && gsz <= L.g && nU >= 0;
    if (!ok)
        set_status(L.status, PW_ERR_INVALID_ARG);
    return ok;
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled operand tile
// (rows of 128 bytes, chunks XOR-swizzled by row % 8, 8-row atoms at 1024 bytes).
__device__ __forceinline__ uint32_t swz(int row, int chunk)
{
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Four E4M3 codes (byte 0 = element 0) -> two bf16x2 words, exactly.  Each byte s.eeee.mmm is
// widened to a 16-bit half whose high byte repeats the sign (prmt sign mode), shifted so that
// eeee.mmm lands in the bf16 exponent/mantissa bits 10..4 with the sign at bit 15; that bf16
// equals the code's value times 2^-120 (subnormal codes included), and one bf16 multiply by
// 2^120 restores it.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t x, uint32_t &lo, uint32_t &hi)
{
    constexpr uint32_t kTwo120 = 0x7B807B80u; // bf16 2^120 in both halves
    const uint32_t a = (prmt(x, 0u, 0x9180u) << 4) & 0x87F087F0u;
    const uint32_t b = (prmt(x, 0u, 0xB3A2u) << 4) & 0x87F087F0u;
    lo = bf16x2_mul(a, kTwo120);
    hi = bf16x2_mul(b, kTwo120);
}

// 64 keys x 128 dims E4M3 (row-major) -> two swizzled 64-dim bf16 blocks.  Thread q handles
// key q/8, dims 16(q%8)..+15 (two 16-byte chunks); threads 4-7 of each quarter-warp store
// their chunks in the opposite order so a quarter-warp's eight stores hit eight bank groups.
template <int NT>
__device__ __forceinline__ void decode_page(const uint8_t *src, uint8_t (*dst)[64 * 128], int tid)
{
#pragma unroll
    for (int rep = 0; rep < 512 / NT; ++rep) {
        const int q = tid + NT * rep;
        const int key = q >> 3, c16 = q & 7;
        const uint4 x = *reinterpret_cast<const uint4 *>(src + key * 128 + c16 * 16);
        uint4 h0, h1;
        e4m3x4_to_bf16x4(x.x, h0.x, h0.y);
        e4m3x4_to_bf16x4(x.y, h0.z, h0.w);
        e4m3x4_to_bf16x4(x.z, h1.x, h1.y);
        e4m3x4_to_bf16x4(x.w, h1.z, h1.w);
        uint8_t *blk = dst[c16 >> 2];
        const int j0 = (2 * c16) & 7;
        if (c16 < 4) {
            *reinterpret_cast<uint4 *>(blk + swz(key, j0)) = h0;
            *reinterpret_cast<uint4 *>(blk + swz(key, j0 + 1)) = h1;
        } else {
            *reinterpret_cast<uint4 *>(blk + swz(key, j0 + 1)) = h1;
            *reinterpret_cast<uint4 *>(blk + swz(key, j0)) = h0;
        }
    }
}

// 64 keys x 128 dims E4M3 (row-major) -> two swizzled 64-dim f16 blocks, the same tile layout
// as decode_page.  E4M3 values are exact in f16 (subnormals included); the hardware converts
// two codes per instruction.
template <int NT>
__device__ __forceinline__ void decode_page_f16(const uint8_t *src, uint8_t (*dst)[64 * 128], int tid)
{
#pragma unroll
    for (int rep = 0; rep < 512 / NT; ++rep) {
        const int q = tid + NT * rep;
        const int key = q >> 3, c16 = q & 7;
        const uint4 x = *reinterpret_cast<const uint4 *>(src + key * 128 + c16 * 16);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\t"
                "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, u;\n\t}\n"
                : "=r"(h[2 * i]), "=r"(h[2 * i + 1])
                : "r"(w[i]));
        const uint4 h0 = make_uint4(h[0], h[1], h[2], h[3]), h1 = make_uint4(h[4], h[5], h[6], h[7]);
        uint8_t *blk = dst[c16 >> 2];
        const int j0 = (2 * c16) & 7;
        if (c16 < 4) {
            *reinterpret_cast<uint4 *>(blk + swz(key, j0)) = h0;
            *reinterpret_cast<uint4 *>(blk + swz(key, j0 + 1)) = h1;
        } else {
            *reinterpret_cast<uint4 *>(blk + swz(key, j0 + 1)) = h1;
            *reinterpret_cast<uint4 *>(blk + swz(key, j0)) = h0;
        }
    }
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// p -> (hi, lo) bf16 halves of two packed words: hi = p rounded to bf16 (round half up on the
// bit pattern), lo = p - hi truncated to bf16.
__device__ __forceinline__ void split_pair(float p0, float p1, uint32_t &hi2, uint32_t &lo2)
{
    const uint32_t u0 = __float_as_uint(p0) + 0x8000u;
    const uint32_t u1 = __float_as_uint(p1) + 0x8000u;
    const float r0 = p0 - __uint_as_float(u0 & 0xFFFF0000u);
    const float r1 = p1 - __uint_as_float(u1 & 0xFFFF0000u);
    hi2 = prmt(u0, u1, 0x7632u);
    lo2 = prmt(__float_as_uint(r0), __float_as_uint(r1), 0x7632u);
}


} // namespace attn
} // namespace pw
