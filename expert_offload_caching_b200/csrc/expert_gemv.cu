// NVFP4 expert GEMV for decode (W4A16): gate/up projection with fused SwiGLU,
// down projection, and the gate-weighted combine.
//
// The routed expert is a SwiGLU FFN over NVFP4 weights (FreeToken pages: routed
// expert MLPs in NVFP4, florigen.ai "NVFP4で約135GBまで縮める"): w = e2m1 * e4m3
// block scale (one per 16 consecutive K) * fp32 tensor scale.
//   h_j = silu(g_j) * u_j,  g = W1 x, u = W3 x;   y_e = W2 h.
//   y = sum over selected e (ascending id) of gate_e * y_e + y_shared.
//
// Decode is HBM-bound (1 row, weights read once).  The kernel streams each
// weight row with 128-bit loads (L1 bypass) and keeps the instruction count
// per byte low enough to stay memory-bound:
//   * E2M1 codes are decoded in registers with cvt.rn.f16x2.e2m1x2 (2 per op);
//   * each fp16 value is multiplied by its E4M3 block scale (cvt.rn.f16x2.e4m3x2);
//     the product of an E2M1 and an E4M3 value is exact in fp16;
//   * the dot products run on the tensor cores (mma.sync m16n8k16, fp16 in,
//     fp32 accumulate): a warp's tile is 16 weight rows, the 8 mma columns
//     carry up to 4 activation rows as fp16 (hi, lo) pairs, hi + lo == the
//     fp32 (or bf16) value, so no precision is lost against fp32 FMAs.
// Each thread owns one 64-element chunk (32 code bytes, 4 scale bytes) of two
// tile rows per K-step; the four threads of an mma quad cover 256 consecutive
// K.  The dot product is order-free, so logical k positions of the mma are
// mapped onto each thread's own chunk, with the activations loaded at the same
// positions.  A CTA of 4 warps splits the K-steps of one tile (or serves 2-4
// tiles when K is short) and reduces in shared memory in a fixed order.
#include "moe_internal.cuh"

namespace moe {

namespace {

__device__ __forceinline__ uint4 ld_stream(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream32(const uint8_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
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
    uint16_t s = (uint16_t)v16;
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

constexpr int kGemvThreads = 128;

template <int NG>
__global__ void __launch_bounds__(kGemvThreads) expert_gemv_kernel(GemvArgs a) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const bool gate_up = a.mode == kGateUp;

    // ---- which expert (job) this CTA serves
    const uint8_t *rec;
    int nrows, row_off = 0;
    bool shared = false;
    if (a.only_job < 0 && (int)blockIdx.y == a.shared_slot) {
        rec = a.shared_rec;
        nrows = a.T;
        shared = true;
    } else {
        const int jy = a.only_job >= 0 ? a.only_job : (int)blockIdx.y;
        if (jy >= *a.n_jobs) return;
        const Job jb = a.jobs[jy];
        if (a.only_job < 0 && !jb.hit) return;
        rec = a.arena + (int64_t)jb.slot * a.rec_bytes;
        nrows = jb.nrows;
        row_off = jb.row_off;
    }

    const int K = gate_up ? a.d : a.F;
    const int NCH = K >> 6;
    const int nsteps = (NCH + 3) >> 2;
    const int tiles = gate_up ? (a.F >> 3) : (a.d >> 4);
    const int tpc = 4 / a.wpt;
    const int tile = blockIdx.x * tpc + warp / a.wpt;
    const int phase = warp % a.wpt;
    const bool active = tile < tiles;

    const int64_t rowA = gate_up ? 2 * (8 * tile + g) : 16 * tile + g;
    const int64_t rowB = gate_up ? rowA + 1 : rowA + 8;
    const uint8_t *codes = rec + (gate_up ? a.lay.w13_codes : a.lay.w2_codes);
    const uint8_t *scales = rec + (gate_up ? a.lay.w13_scales : a.lay.w2_scales);
    const uint8_t *cA = codes + rowA * (K >> 1), *cB = codes + rowB * (K >> 1);
    const uint8_t *sA = scales + rowA * (K >> 4), *sB = scales + rowB * (K >> 4);
    const float *ts = reinterpret_cast<const float *>(rec + a.lay.tscales);

    __shared__ float red[4][NG][4][32];

    for (int r0 = 0; r0 < nrows; r0 += 4 * NG) {
        // B-operand column of this thread: mma column n = g carries activation row
        // r0 + 4*grp + g/2, the hi (g even) or lo (g odd) fp16 part.
        const __half *col[NG];
        bool colv[NG];
        int ngrp = 0;
#pragma unroll
        for (int grp = 0; grp < NG; ++grp) {
            const int r = r0 + 4 * grp + (g >> 1);
            colv[grp] = active && r < nrows;
            col[grp] = a.act;
            if (r0 + 4 * grp < nrows) ngrp = grp + 1;
            if (colv[grp]) {
                int t, p;
                if (shared) { t = r; p = a.k; }
                else { RowRef rr = a.rowrefs[row_off + r]; t = rr.t; p = rr.p; }
                col[grp] = gate_up ? a.act + (size_t)t * 2 * a.d + (g & 1) * a.d
                                   : a.act + (size_t)(t * (a.k + 1) + p) * 2 * a.F + (g & 1) * a.F;
            }
        }

        float acc[NG][4];
#pragma unroll
        for (int grp = 0; grp < NG; ++grp)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[grp][j] = 0.f;

        if (active) {
            for (int s = phase; s < nsteps; s += a.wpt) {
                const int c = 4 * s + q;
                const bool cv = c < NCH;
                uint4 qa0 = make_uint4(0, 0, 0, 0), qa1 = qa0, qb0 = qa0, qb1 = qa0;
                uint32_t sca = 0, scb = 0;
                if (cv) {
                    qa0 = ld_stream(cA + 32 * c);
                    qa1 = ld_stream(cA + 32 * c + 16);
                    qb0 = ld_stream(cB + 32 * c);
                    qb1 = ld_stream(cB + 32 * c + 16);
                    sca = ld_stream32(sA + 4 * c);
                    scb = ld_stream32(sB + 4 * c);
                }
                const __half2 a01 = e4m3x2_to_h2(sca & 0xffffu), a23 = e4m3x2_to_h2(sca >> 16);
                const __half2 b01 = e4m3x2_to_h2(scb & 0xffffu), b23 = e4m3x2_to_h2(scb >> 16);
                const __half2 sAv[4] = {__low2half2(a01), __high2half2(a01), __low2half2(a23),
                                        __high2half2(a23)};
                const __half2 sBv[4] = {__low2half2(b01), __high2half2(b01), __low2half2(b23),
                                        __high2half2(b23)};
                const uint32_t wa[8] = {qa0.x, qa0.y, qa0.z, qa0.w, qa1.x, qa1.y, qa1.z, qa1.w};
                const uint32_t wb[8] = {qb0.x, qb0.y, qb0.z, qb0.w, qb1.x, qb1.y, qb1.z, qb1.w};
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    uint32_t fa[4], fb[4];
                    e2m1x8_to_f16(wa[w], fa);
                    e2m1x8_to_f16(wb[w], fb);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        fa[j] = hmul2u(fa[j], sAv[w >> 1]);
                        fb[j] = hmul2u(fb[j], sBv[w >> 1]);
                    }
#pragma unroll
                    for (int grp = 0; grp < NG; ++grp) {
                        if (grp < ngrp) {
                            uint4 bv = make_uint4(0, 0, 0, 0);
                            if (colv[grp] && cv)
                                bv = __ldg(reinterpret_cast<const uint4 *>(col[grp] + 64 * c + 8 * w));
                            mma16816(acc[grp], fa[0], fb[0], fa[1], fb[1], bv.x, bv.y);
                            mma16816(acc[grp], fa[2], fb[2], fa[3], fb[3], bv.z, bv.w);
                        }
                    }
                }
            }
        }

        // ---- reduce the K-split warps of a tile (fixed order), then the epilogue
        if (a.wpt > 1) {
#pragma unroll
            for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                for (int j = 0; j < 4; ++j) red[warp][grp][j][lane] = acc[grp][j];
            __syncthreads();
            if (phase == 0) {
                for (int ph = 1; ph < a.wpt; ++ph)
#pragma unroll
                    for (int grp = 0; grp < NG; ++grp)
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc[grp][j] += red[warp + ph][grp][j][lane];
            }
            __syncthreads();
        }
        if (active && phase == 0) {
#pragma unroll
            for (int grp = 0; grp < NG; ++grp) {
                const int r = r0 + 4 * grp + q;  // this thread's results: activation row q
                if (r >= nrows) continue;
                int t, p;
                if (shared) { t = r; p = a.k; }
                else { RowRef rr = a.rowrefs[row_off + r]; t = rr.t; p = rr.p; }
                const float v0 = acc[grp][0] + acc[grp][1];  // tile row g
                const float v1 = acc[grp][2] + acc[grp][3];  // tile row g + 8
                const size_t sel = (size_t)t * (a.k + 1) + p;
                if (gate_up) {
                    const float gt = ts[0] * v0, up = ts[1] * v1;
                    const float h = gt / (1.0f + expf(-gt)) * up;
                    const __half hi = __float2half_rn(h);
                    const __half lo = __float2half_rn(h - __half2float(hi));
                    const int j = 8 * tile + g;
                    a.hh_out[sel * 2 * a.F + j] = hi;
                    a.hh_out[sel * 2 * a.F + a.F + j] = lo;
                } else {
                    const int i = 16 * tile + g;
                    a.part_out[sel * a.d + i] = ts[2] * v0;
                    a.part_out[sel * a.d + i + 8] = ts[2] * v1;
                }
            }
        }
    }
}

__global__ void combine_kernel(const float *__restrict__ part, const float *__restrict__ gates,
                               float *__restrict__ y, int T, int k, int d, int has_shared) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * d) return;
    const int t = i / d, c = i - t * d;
    const float *pr = part + (size_t)t * (k + 1) * d + c;
    float acc = 0.f;
    for (int p = 0; p < k; ++p) acc = fmaf(gates[t * k + p], pr[(size_t)p * d], acc);
    if (has_shared) acc += pr[(size_t)k * d];
    y[i] = acc;
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs &a, int grid_y, cudaStream_t s) {
    const int tiles = a.mode == kGateUp ? a.F / 8 : a.d / 16;
    const int tpc = 4 / a.wpt;
    dim3 grid((tiles + tpc - 1) / tpc, grid_y);
    const int rows = a.T;
    if (rows <= 4) expert_gemv_kernel<1><<<grid, kGemvThreads, 0, s>>>(a);
    else if (rows <= 8) expert_gemv_kernel<2><<<grid, kGemvThreads, 0, s>>>(a);
    else expert_gemv_kernel<4><<<grid, kGemvThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_combine(const float *part, const float *gates, float *y, int T, int k, int d,
                           int has_shared, cudaStream_t s) {
    const int n = T * d;
    combine_kernel<<<(n + 255) / 256, 256, 0, s>>>(part, gates, y, T, k, d, has_shared);
    return cudaGetLastError();
}

}  // namespace moe
