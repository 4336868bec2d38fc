// sru_attention.cuh -- the row-wise steps of SRU++'s attention producer of U.
//
// "When Attention Meets Fast Recurrence" (SRU++ section): SRU++ replaces the
// linear map of Eq. (1) by single-head attention over d' = d/4 features,
//   Q = W_q X^T,  K = W_k Q,  V = W_v Q,
//   A^T = softmax(Q^T K / sqrt(d')) V^T,
//   U^T = W_o (Q + alpha A)      or  W_o layernorm(Q + alpha A)
// (post-attention normalisation).  The products run on the tensor-core GEMM
// (sru_gemm.cuh); this file holds the two row-wise steps between them: the
// scaled, optionally causal softmax of one batch row's L x L scores, and the
// residual Q + alpha A with the optional layer norm.  One warp per row.
#pragma once

#include <cuda_bf16.h>

#include "sru_ptx.cuh"

namespace sru {

constexpr int kRowWarps = 8;  // rows per CTA
constexpr float kLayerNormEps = 1e-5f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// P[t][s] = exp(z_s - max) / sum over the visible s of exp(z - max), with
// z_s = S[t][s] * scale; visible: s <= t when causal, else all s < L.
// Invisible entries of P are written as 0.  S (rows / L, L, L) fp32 holds
// rows / L batch rows' score matrices back to back; P likewise in bf16.
__global__ void __launch_bounds__(kRowWarps * 32) sru_softmax_rows_kernel(const float* __restrict__ S,
                                                                        __nv_bfloat16* __restrict__ P, int L,
                                                                        int rows, float scale, int causal) {
    const int row = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int t = row % L;
    const float* srow = S + (size_t)row * L;
    __nv_bfloat16* prow = P + (size_t)row * L;
    const int n = causal ? t + 1 : L;
    float m = -INFINITY;
    for (int s = lane; s < n; s += 32) m = fmaxf(m, srow[s] * scale);
    m = warp_max(m);
    float sum = 0.f;
    for (int s = lane; s < n; s += 32) sum += expf(srow[s] * scale - m);
    const float inv = 1.0f / warp_sum(sum);
    for (int s = lane; s < L; s += 32)
        prow[s] = __float2bfloat16_rn(s < n ? expf(srow[s] * scale - m) * inv : 0.f);
}

// R[m][j] = bf16(z) with z = Q[m][j] + alpha * A[m][j], or, with gamma/beta,
// bf16((z - mean_j z) / sqrt(var_j z + eps) * gamma[j] + beta[j]) over the
// d' features of row m (two passes for the mean and the variance).
__global__ void __launch_bounds__(kRowWarps * 32) sru_residual_norm_kernel(
    const __nv_bfloat16* __restrict__ Q, const float* __restrict__ A, float alpha, const float* __restrict__ gamma,
    const float* __restrict__ beta, __nv_bfloat16* __restrict__ R, int M, int dp) {
    const int m = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (m >= M) return;
    const __nv_bfloat16* q = Q + (size_t)m * dp;
    const float* a = A + (size_t)m * dp;
    __nv_bfloat16* r = R + (size_t)m * dp;
    if (gamma == nullptr) {
        for (int j = lane; j < dp; j += 32) r[j] = __float2bfloat16_rn(fmaf(alpha, a[j], __bfloat162float(q[j])));
        return;
    }
    float sum = 0.f;
    for (int j = lane; j < dp; j += 32) sum += fmaf(alpha, a[j], __bfloat162float(q[j]));
    const float mean = warp_sum(sum) / (float)dp;
    float sq = 0.f;
    for (int j = lane; j < dp; j += 32) {
        const float z = fmaf(alpha, a[j], __bfloat162float(q[j])) - mean;
        sq = fmaf(z, z, sq);
    }
    const float rstd = rsqrtf(warp_sum(sq) / (float)dp + kLayerNormEps);
    for (int j = lane; j < dp; j += 32) {
        const float z = fmaf(alpha, a[j], __bfloat162float(q[j])) - mean;
        r[j] = __float2bfloat16_rn(fmaf(z * rstd, gamma[j], beta[j]));
    }
}

}  // namespace sru
