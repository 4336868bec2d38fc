// sru_decode.cuh -- one time step of the SRU layer for token-by-token
// inference, with the projection fused in.
//
// "When Attention Meets Fast Recurrence" (background section on SRU) notes
// that an SRU model runs as an RNN at inference time.  Per step, Eq. (1)
// becomes a matrix-vector product u = W_cat x_t (per batch row) and
// Eqs. (2)-(5) one cell update.  The product streams all of W_cat (6 d^2
// bytes) for a handful of flops per byte, so the step is bound by HBM reads of
// W; u never needs to exist in memory.
//
// Layout of the work: one warp per hidden channel j.  The warp reads the
// three rows of W_cat that feed channel j (candidate, forget, reset) with
// 16-byte loads that bypass L1 (each element is used once per call), dots
// them with up to NB batch rows of X_t, reduces the 3*NB sums across the
// warp, and lanes b < NB apply the cell to (b, j).
#pragma once

#include "sru_recurrence.cuh"

namespace sru {

constexpr int kDecWarps = 8;  // channels per CTA
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecMaxNB = 16;  // batch rows per pass over W

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 8 bf16 (one 16-byte word) -> 8 fp32 (exact)
__device__ __forceinline__ void unpack8(const uint4& w, float (&o)[8]) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(a[i] << 16);
        o[2 * i + 1] = __uint_as_float(a[i] & 0xFFFF0000u);
    }
}

// Eqs. (2)-(5) for one element, the same operations in the same order as
// sru_cell2 and the forward's h (so a decode step and a forward step agree
// bit for bit when given the same u).
__device__ __forceinline__ float sru_cell1(float c, float uc, float uf, float ur, float vf, float vr, float bf,
                                           float br, float ax, float& h) {
    const float nvf = __fmul_rn(vf, kNegLog2e), nvr = __fmul_rn(vr, kNegLog2e);
    const float nbf = __fmul_rn(bf, kNegLog2e), nbr = __fmul_rn(br, kNegLog2e);
    const float f = sigmoid_nl2(__fmaf_rn(nvf, c, __fmaf_rn(uf, kNegLog2e, nbf)));
    const float r = sigmoid_nl2(__fmaf_rn(nvr, c, __fmaf_rn(ur, kNegLog2e, nbr)));
    const float cn = __fmaf_rn(f, __fmaf_rn(uc, -1.0f, c), uc);
    h = __fmaf_rn(r, __fmaf_rn(ax, -1.0f, cn), ax);
    return cn;
}

// Grid (ceil(d / kDecWarps), ceil(B / NB)); no shared memory.  Everything a
// warp needs besides W (its X rows, which every warp reads and L1 keeps, and
// the cell operands of channel j) is fetched before or alongside the W stream,
// so a step costs one pass over W plus one load latency.
template <int NB>
__global__ void __launch_bounds__(kDecThreads) sru_decode_step_kernel(
    const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ W, const float* __restrict__ x,
    const float* __restrict__ v, const float* __restrict__ bias, float* __restrict__ c, float* __restrict__ h,
    int B, int d, float alpha) {
    constexpr int kUnroll = NB >= 8 ? 2 : 4;  // W words in flight per lane and gate (register budget)
    const int b0 = blockIdx.y * NB;
    const int nb = min(NB, B - b0);
    const int kw = d / 8;  // 16-byte words per row (d % 8 == 0)
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int j = blockIdx.x * kDecWarps + warp;
    if (j >= d) return;

    // cell operands: lane bb < nb owns batch row b0 + bb of channel j
    const size_t e = (size_t)(b0 + min(lane, nb - 1)) * d + j;
    const float c_in = c[e], ax = __fmul_rn(alpha, x[e]);
    const float vf = v[j], vr = v[d + j], bf = bias[j], br = bias[d + j];

    float acc[3][NB];
#pragma unroll
    for (int g = 0; g < 3; ++g)
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) acc[g][bb] = 0.f;

    const uint4* w0 = reinterpret_cast<const uint4*>(W + (size_t)j * d);
    const uint4* w1 = reinterpret_cast<const uint4*>(W + (size_t)(d + j) * d);
    const uint4* w2 = reinterpret_cast<const uint4*>(W + (size_t)(2 * d + j) * d);
    const uint4* Xw = reinterpret_cast<const uint4*>(X) + (size_t)b0 * kw;
#pragma unroll kUnroll
    for (int k = lane; k < kw; k += 32) {
        float wc[8], wf[8], wr[8];
        unpack8(ld_stream_u4(w0 + k), wc);
        unpack8(ld_stream_u4(w1 + k), wf);
        unpack8(ld_stream_u4(w2 + k), wr);
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) {
            float xv[8];
            unpack8(__ldg(Xw + (size_t)min(bb, nb - 1) * kw + k), xv);  // rows past nb: unused
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                acc[0][bb] = __fmaf_rn(wc[q], xv[q], acc[0][bb]);
                acc[1][bb] = __fmaf_rn(wf[q], xv[q], acc[1][bb]);
                acc[2][bb] = __fmaf_rn(wr[q], xv[q], acc[2][bb]);
            }
        }
    }
    // every lane ends with all 3*NB sums
#pragma unroll
    for (int g = 0; g < 3; ++g)
#pragma unroll
        for (int bb = 0; bb < NB; ++bb)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[g][bb] += __shfl_xor_sync(0xffffffffu, acc[g][bb], o);

    // lane bb updates batch row b0 + bb (register indices must be compile-time)
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) {
        if (lane != bb || bb >= nb) continue;
        float hv;
        c[e] = sru_cell1(c_in, acc[0][bb], acc[1][bb], acc[2][bb], vf, vr, bf, br, ax, hv);
        h[e] = hv;
    }
}

// Batched decoding (B rows per step): u = W_cat X_t^T has been computed on the
// tensor cores into u (3d x B fp32, row g*d + j, column b); this applies
// Eqs. (2)-(5) to every (b, j) with the same operations as sru_cell1.
// One thread per (j, b), b fastest (consecutive threads read consecutive u).
__global__ void __launch_bounds__(256) sru_decode_cell_kernel(const float* __restrict__ u,
                                                              const float* __restrict__ x,
                                                              const float* __restrict__ v,
                                                              const float* __restrict__ bias,
                                                              float* __restrict__ c, float* __restrict__ h, int B,
                                                              int d, float alpha) {
    const size_t i = (size_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= (size_t)B * d) return;
    const int b = (int)(i % B), j = (int)(i / B);
    const float uc = u[(size_t)j * B + b], uf = u[((size_t)d + j) * B + b], ur = u[((size_t)2 * d + j) * B + b];
    const size_t e = (size_t)b * d + j;
    float hv;
    c[e] = sru_cell1(c[e], uc, uf, ur, v[j], v[d + j], bias[j], bias[d + j], __fmul_rn(alpha, x[e]), hv);
    h[e] = hv;
}

}  // namespace sru
