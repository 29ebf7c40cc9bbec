// Inner loops of the decode expert GEMVs (NVFP4 / MXFP4 weights, fp16 (hi, lo)
// activations, mma.sync m16n8k16 with fp32 accumulation), shared by the
// per-launch GEMV kernel and the persistent layer kernel.
#pragma once
#include "moe_internal.cuh"

namespace moe {
namespace gemv {

// Activation fragment load: read-only path (data from an earlier kernel) or
// L2 (data another CTA of the same kernel wrote: the read-only path may not
// see it).
template <bool kCg>
__device__ __forceinline__ uint4 ld_act(const __half *p) {
    if constexpr (kCg) return __ldcg(reinterpret_cast<const uint4 *>(p));
    else return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Prefetch [p, p + bytes) into L2, one 128-byte line per thread of the CTA.
__device__ __forceinline__ void prefetch_l2_range(const uint8_t *p, uint32_t bytes) {
    for (uint32_t o = threadIdx.x * 128u; o < bytes; o += blockDim.x * 128u)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p + o));
}

// 8 E2M1 codes (one 32-bit word, element 2i in the low nibble of byte i) ->
// 4 f16x2 registers {element 2i (low half), 2i+1 (high half)}.
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

__device__ __forceinline__ __half2 e4m3x2_to_h2(uint32_t v16) {
    uint32_t r;
    const uint16_t s = (uint16_t)v16;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(s));
    return *reinterpret_cast<__half2 *>(&r);
}

__device__ __forceinline__ uint32_t hmul2u(uint32_t a, __half2 s) {
    __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&a), s);
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^diff + kMxBias as an fp16 pair (diff <= 0: an E8M0 code minus the largest
// code of its K-step; 0 below the fp16 range).
constexpr int kMxBias = 12;
__device__ __forceinline__ __half2 mx_pow2_h2(int diff) {
    const int e = diff + kMxBias;  // <= 12
    uint32_t bits = e >= -14 ? (uint32_t)(e + 15) << 10 : (e >= -24 ? 1u << (e + 24) : 0u);
    bits |= bits << 16;
    return *reinterpret_cast<__half2 *>(&bits);
}
// 2^(code - 127 - kMxBias) in fp32 (code 255, E8M0's NaN: NaN).
__device__ __forceinline__ float mx_factor(int code) {
    if (code == 255) return __int_as_float(0x7fc00000);
    const int b = code - kMxBias;  // the fp32 biased exponent
    return __int_as_float(b >= 1 ? b << 23 : 1 << (b + 22));
}

// MXFP4 K-step of one thread: as step_mma, with sa / sb holding the two E8M0
// codes (blocks of 32) of the thread's chunk of rows rA / rB.  The mma
// accumulates into a zeroed step sum, which is scaled by 2^(c_max - 139) per
// row (c_max over the quad's chunks, so over the whole mma row) and added.
template <int NG, bool kCg = false>
__device__ __forceinline__ void step_mma_mx(const uint8_t *cA, const uint8_t *cB, uint32_t sa, uint32_t sb,
                                            int c, bool cv, const __half *const (&col)[NG],
                                            const bool (&colv)[NG], int ngrp, float (&acc)[NG][4]) {
    const int a0 = sa & 0xff, a1 = (sa >> 8) & 0xff, b0 = sb & 0xff, b1 = (sb >> 8) & 0xff;
    int ma = max(a0, a1), mb = max(b0, b1);
    ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
    ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
    const __half2 sAv[2] = {mx_pow2_h2(a0 - ma), mx_pow2_h2(a1 - ma)};
    const __half2 sBv[2] = {mx_pow2_h2(b0 - mb), mx_pow2_h2(b1 - mb)};
    float stp[NG][4];
#pragma unroll
    for (int grp = 0; grp < NG; ++grp)
#pragma unroll
        for (int i = 0; i < 4; ++i) stp[grp][i] = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 qa = cv ? *reinterpret_cast<const uint4 *>(cA + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint4 qb = cv ? *reinterpret_cast<const uint4 *>(cB + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
        const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int w = 4 * h + u;  // 8 codes: elements 8w .. 8w+7 of the chunk, block w / 4
            uint32_t fa[4], fb[4];
            e2m1x8_to_f16(wa[u], fa);
            e2m1x8_to_f16(wb[u], fb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                fa[j] = hmul2u(fa[j], sAv[w >> 2]);
                fb[j] = hmul2u(fb[j], sBv[w >> 2]);
            }
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                if (grp < ngrp) {
                    uint4 bv = make_uint4(0, 0, 0, 0);
                    if (colv[grp] && cv) bv = ld_act<kCg>(col[grp] + 64 * c + 8 * w);
                    mma16816(stp[grp], fa[0], fb[0], fa[1], fb[1], bv.x, bv.y);
                    mma16816(stp[grp], fa[2], fb[2], fa[3], fb[3], bv.z, bv.w);
                }
            }
        }
    }
    const float fA = mx_factor(ma), fB = mx_factor(mb);
#pragma unroll
    for (int grp = 0; grp < NG; ++grp) {  // d0, d1: row rA; d2, d3: row rB
        acc[grp][0] = fmaf(stp[grp][0], fA, acc[grp][0]);
        acc[grp][1] = fmaf(stp[grp][1], fA, acc[grp][1]);
        acc[grp][2] = fmaf(stp[grp][2], fB, acc[grp][2]);
        acc[grp][3] = fmaf(stp[grp][3], fB, acc[grp][3]);
    }
}

constexpr int kMaxSteps = 16;  // K <= 4096: at most 16 K-steps of 256, one per warp
constexpr int kGStages = 3;                           // tiles in flight per CTA

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
// L2 policy for data read once (expert weights streamed through a layer):
// evict it first, so that what the next steps reuse -- the routers, the cache
// table, the activations -- stays in L2.
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void cp_async16_ef(void *dst, const void *src, uint64_t policy) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "l"(policy)
                 : "memory");
}
// 16-byte asynchronous copy global -> shared (L1 bypassed), tracked per thread.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

// One K-step of one thread: 32 code bytes of each of its two tile rows (from
// shared memory) and their 4 scale bytes each.  cv = false (the chunk lies past
// the end of K) feeds zeros.  Every lane of the warp must call this together:
// mma.sync is a warp-collective (.aligned) instruction.
template <int NG, bool kCg = false>
__device__ __forceinline__ void step_mma(const uint8_t *cA, const uint8_t *cB, uint32_t sa, uint32_t sb,
                                         int c, bool cv, const __half *const (&col)[NG],
                                         const bool (&colv)[NG], int ngrp, float (&acc)[NG][4]) {
    const __half2 a01 = e4m3x2_to_h2(sa & 0xffffu), a23 = e4m3x2_to_h2(sa >> 16);
    const __half2 b01 = e4m3x2_to_h2(sb & 0xffffu), b23 = e4m3x2_to_h2(sb >> 16);
    const __half2 sAv[4] = {__low2half2(a01), __high2half2(a01), __low2half2(a23), __high2half2(a23)};
    const __half2 sBv[4] = {__low2half2(b01), __high2half2(b01), __low2half2(b23), __high2half2(b23)};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 qa = cv ? *reinterpret_cast<const uint4 *>(cA + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint4 qb = cv ? *reinterpret_cast<const uint4 *>(cB + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
        const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int w = 4 * h + u;  // 8 codes: elements 8w .. 8w+7 of the chunk
            uint32_t fa[4], fb[4];
            e2m1x8_to_f16(wa[u], fa);
            e2m1x8_to_f16(wb[u], fb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                fa[j] = hmul2u(fa[j], sAv[w >> 1]);
                fb[j] = hmul2u(fb[j], sBv[w >> 1]);
            }
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                if (grp < ngrp) {
                    uint4 bv = make_uint4(0, 0, 0, 0);
                    if (colv[grp] && cv) bv = ld_act<kCg>(col[grp] + 64 * c + 8 * w);
                    mma16816(acc[grp], fa[0], fb[0], fa[1], fb[1], bv.x, bv.y);
                    mma16816(acc[grp], fa[2], fb[2], fa[3], fb[3], bv.z, bv.w);
                }
            }
        }
    }
}

// Activation fragment load, three ways: 0 read-only path (data from an earlier
// kernel), 1 L2 (written by another CTA of this kernel), 2 shared memory (the
// pointer is into this CTA's shared memory).
template <int kAct>
__device__ __forceinline__ uint4 ld_act3(const __half *p) {
    if constexpr (kAct == 0) return __ldg(reinterpret_cast<const uint4 *>(p));
    else if constexpr (kAct == 1) return __ldcg(reinterpret_cast<const uint4 *>(p));
    else return *reinterpret_cast<const uint4 *>(p);
}

// step_mma / step_mma_mx with two accumulator sets: the first 32 codes of the
// chunk (h = 0) go into acc0, the last 32 (h = 1) into acc1, so the mma
// dependency chain is half as long (the dot product is order-free).
template <int NG, int kAct = 0>
__device__ __forceinline__ void step_mma_x2(const uint8_t *cA, const uint8_t *cB, uint32_t sa, uint32_t sb, int c,
                                            bool cv, const __half *const (&col)[NG], const bool (&colv)[NG], int ngrp,
                                            float (&acc0)[NG][4], float (&acc1)[NG][4]) {
    const __half2 a01 = e4m3x2_to_h2(sa & 0xffffu), a23 = e4m3x2_to_h2(sa >> 16);
    const __half2 b01 = e4m3x2_to_h2(sb & 0xffffu), b23 = e4m3x2_to_h2(sb >> 16);
    const __half2 sAv[4] = {__low2half2(a01), __high2half2(a01), __low2half2(a23), __high2half2(a23)};
    const __half2 sBv[4] = {__low2half2(b01), __high2half2(b01), __low2half2(b23), __high2half2(b23)};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float(&acc)[NG][4] = h == 0 ? acc0 : acc1;
        const uint4 qa = cv ? *reinterpret_cast<const uint4 *>(cA + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint4 qb = cv ? *reinterpret_cast<const uint4 *>(cB + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
        const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int w = 4 * h + u;
            uint32_t fa[4], fb[4];
            e2m1x8_to_f16(wa[u], fa);
            e2m1x8_to_f16(wb[u], fb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                fa[j] = hmul2u(fa[j], sAv[w >> 1]);
                fb[j] = hmul2u(fb[j], sBv[w >> 1]);
            }
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                if (grp < ngrp) {
                    uint4 bv = make_uint4(0, 0, 0, 0);
                    if (colv[grp] && cv) bv = ld_act3<kAct>(col[grp] + 64 * c + 8 * w);
                    mma16816(acc[grp], fa[0], fb[0], fa[1], fb[1], bv.x, bv.y);
                    mma16816(acc[grp], fa[2], fb[2], fa[3], fb[3], bv.z, bv.w);
                }
            }
        }
    }
}

template <int NG, int kAct = 0>
__device__ __forceinline__ void step_mma_mx_x2(const uint8_t *cA, const uint8_t *cB, uint32_t sa, uint32_t sb, int c,
                                               bool cv, const __half *const (&col)[NG], const bool (&colv)[NG],
                                               int ngrp, float (&acc0)[NG][4], float (&acc1)[NG][4]) {
    const int a0 = sa & 0xff, a1 = (sa >> 8) & 0xff, b0 = sb & 0xff, b1 = (sb >> 8) & 0xff;
    int ma = max(a0, a1), mb = max(b0, b1);
    ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
    ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
    mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
    const __half2 sAv[2] = {mx_pow2_h2(a0 - ma), mx_pow2_h2(a1 - ma)};
    const __half2 sBv[2] = {mx_pow2_h2(b0 - mb), mx_pow2_h2(b1 - mb)};
    float stp[2][NG][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int grp = 0; grp < NG; ++grp)
#pragma unroll
            for (int i = 0; i < 4; ++i) stp[h][grp][i] = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 qa = cv ? *reinterpret_cast<const uint4 *>(cA + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint4 qb = cv ? *reinterpret_cast<const uint4 *>(cB + 16 * h) : make_uint4(0, 0, 0, 0);
        const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
        const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int w = 4 * h + u;  // block w / 4 == h
            uint32_t fa[4], fb[4];
            e2m1x8_to_f16(wa[u], fa);
            e2m1x8_to_f16(wb[u], fb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                fa[j] = hmul2u(fa[j], sAv[h]);
                fb[j] = hmul2u(fb[j], sBv[h]);
            }
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                if (grp < ngrp) {
                    uint4 bv = make_uint4(0, 0, 0, 0);
                    if (colv[grp] && cv) bv = ld_act3<kAct>(col[grp] + 64 * c + 8 * w);
                    mma16816(stp[h][grp], fa[0], fb[0], fa[1], fb[1], bv.x, bv.y);
                    mma16816(stp[h][grp], fa[2], fb[2], fa[3], fb[3], bv.z, bv.w);
                }
            }
        }
    }
    const float fA = mx_factor(ma), fB = mx_factor(mb);
#pragma unroll
    for (int grp = 0; grp < NG; ++grp) {  // d0, d1: row rA; d2, d3: row rB
        acc0[grp][0] = fmaf(stp[0][grp][0], fA, acc0[grp][0]);
        acc0[grp][1] = fmaf(stp[0][grp][1], fA, acc0[grp][1]);
        acc0[grp][2] = fmaf(stp[0][grp][2], fB, acc0[grp][2]);
        acc0[grp][3] = fmaf(stp[0][grp][3], fB, acc0[grp][3]);
        acc1[grp][0] = fmaf(stp[1][grp][0], fA, acc1[grp][0]);
        acc1[grp][1] = fmaf(stp[1][grp][1], fA, acc1[grp][1]);
        acc1[grp][2] = fmaf(stp[1][grp][2], fB, acc1[grp][2]);
        acc1[grp][3] = fmaf(stp[1][grp][3], fB, acc1[grp][3]);
    }
}

}  // namespace gemv
}  // namespace moe
