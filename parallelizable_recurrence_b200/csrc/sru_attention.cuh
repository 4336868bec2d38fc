// sru_attention.cuh -- the row-wise steps of SRU++'s attention producer of U.
//
// "When Attention Meets Fast Recurrence" (SRU++ section): SRU++ replaces the
// linear map of Eq. (1) by single-head attention over d' = d/4 features,
//   Q = W_q X^T,  K = W_k Q,  V = W_v Q,
//   A^T = softmax(Q^T K / sqrt(d')) V^T,
//   U^T = W_o (Q + alpha A)      or  W_o layernorm(Q + alpha A)
// (post-attention normalisation).  The products run on the tensor-core GEMM
// (sru_gemm.cuh); this file holds the row-wise steps between them: the
// scaled, optionally causal softmax of one batch row's L x L scores, and the
// residual Q + alpha A with the optional layer norm, and, for the backward
// (the reverse-mode derivative of those two steps), the softmax's and the
// norm's gradients.  One warp per row, except the column sums of the norm's
// parameter gradients.
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

// The same softmax with the row held in registers (rows of at most NV * 128
// scores, read once with 16-byte loads): lane l owns scores 4l .. 4l + 3 of
// every 128.  When causal, P is written only up to the end of the row's
// 256-wide tile: the products that read P (P V up to the end of each row
// tile, P^T dA from each row tile's diagonal on) never read further.
template <int NV>
__global__ void __launch_bounds__(kRowWarps * 32) sru_softmax_rows_reg_kernel(const float* __restrict__ S,
                                                                            __nv_bfloat16* __restrict__ P, int L,
                                                                            int rows, float scale, int causal) {
    const int row = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int t = row % L;
    const float4* srow = reinterpret_cast<const float4*>(S + (size_t)row * L);
    uint2* prow = reinterpret_cast<uint2*>(P + (size_t)row * L);
    const int n = causal ? t + 1 : L;
    const int end = causal ? min(L, (t / 256 + 1) * 256) : L;  // written: [0, end)
    float4 v[NV];
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int s0 = k * 128 + lane * 4;
        v[k] = s0 < n ? srow[s0 / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
        v[k].x = s0 + 0 < n ? v[k].x * scale : -INFINITY;
        v[k].y = s0 + 1 < n ? v[k].y * scale : -INFINITY;
        v[k].z = s0 + 2 < n ? v[k].z * scale : -INFINITY;
        v[k].w = s0 + 3 < n ? v[k].w * scale : -INFINITY;
        m = fmaxf(m, fmaxf(fmaxf(v[k].x, v[k].y), fmaxf(v[k].z, v[k].w)));
    }
    m = warp_max(m);
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        v[k].x = expf(v[k].x - m);
        v[k].y = expf(v[k].y - m);
        v[k].z = expf(v[k].z - m);
        v[k].w = expf(v[k].w - m);
        sum += (v[k].x + v[k].y) + (v[k].z + v[k].w);
    }
    const float inv = 1.0f / warp_sum(sum);
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int s0 = k * 128 + lane * 4;
        if (s0 >= end) continue;
        __nv_bfloat162 lo = __floats2bfloat162_rn(v[k].x * inv, v[k].y * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(v[k].z * inv, v[k].w * inv);
        prow[s0 / 4] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
}

// The residual and norm with the row held in registers (d' at most NV * 128,
// read once): lane l owns features 4l .. 4l + 3 of every 128.  gamma and beta
// are read 16 bytes at a time.
template <int NV>
__global__ void __launch_bounds__(kRowWarps * 32) sru_residual_norm_reg_kernel(
    const __nv_bfloat16* __restrict__ Q, const float* __restrict__ A, float alpha, const float* __restrict__ gamma,
    const float* __restrict__ beta, __nv_bfloat16* __restrict__ R, int M, int dp) {
    const int m = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (m >= M) return;
    const uint2* q = reinterpret_cast<const uint2*>(Q + (size_t)m * dp);
    const float4* a = reinterpret_cast<const float4*>(A + (size_t)m * dp);
    uint2* r = reinterpret_cast<uint2*>(R + (size_t)m * dp);
    float z[NV][4];
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int j0 = k * 128 + lane * 4;
        if (j0 < dp) {
            const uint2 qq = q[j0 / 4];
            const float4 aa = a[j0 / 4];
            const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qq.x));
            const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qq.y));
            z[k][0] = fmaf(alpha, aa.x, q01.x);
            z[k][1] = fmaf(alpha, aa.y, q01.y);
            z[k][2] = fmaf(alpha, aa.z, q23.x);
            z[k][3] = fmaf(alpha, aa.w, q23.y);
            sum += z[k][0] + z[k][1] + z[k][2] + z[k][3];
        } else {
            z[k][0] = z[k][1] = z[k][2] = z[k][3] = 0.f;
        }
    }
    float mean = 0.f, rstd = 1.f;
    if (gamma != nullptr) {
        mean = warp_sum(sum) / (float)dp;
        float sq = 0.f;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            if (k * 128 + lane * 4 >= dp) continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) sq = fmaf(z[k][e] - mean, z[k][e] - mean, sq);
        }
        rstd = rsqrtf(warp_sum(sq) / (float)dp + kLayerNormEps);
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int j0 = k * 128 + lane * 4;
        if (j0 >= dp) continue;
        float o[4];
        if (gamma == nullptr) {
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = z[k][e];
        } else {
            const float4 g4 = *reinterpret_cast<const float4*>(gamma + j0);
            const float4 b4 = *reinterpret_cast<const float4*>(beta + j0);
            o[0] = fmaf((z[k][0] - mean) * rstd, g4.x, b4.x);
            o[1] = fmaf((z[k][1] - mean) * rstd, g4.y, b4.y);
            o[2] = fmaf((z[k][2] - mean) * rstd, g4.z, b4.z);
            o[3] = fmaf((z[k][3] - mean) * rstd, g4.w, b4.w);
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]), hi = __floats2bfloat162_rn(o[2], o[3]);
        r[j0 / 4] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
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

// ------------------------------------------------------------------ backward
// Softmax gradient of one row t: with p = P[t][.] (the bf16 probabilities the
// forward multiplied by V) and g = dP[t][.],
//   dS[t][s] = p_s (g_s - sum_s' p_s' g_s') * scale       for the visible s,
// and 0 for the others (so that products reading up to the end of a row's
// tile see zeros).  The scale is the forward's 1/sqrt(d'): the scores'
// gradient is taken with respect to Q K^T itself.
__global__ void __launch_bounds__(kRowWarps * 32) sru_softmax_backward_rows_kernel(
    const float* __restrict__ dP, const __nv_bfloat16* __restrict__ P, __nv_bfloat16* __restrict__ dS, int L, int rows,
    float scale, int causal) {
    const int row = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int t = row % L;
    const float* grow = dP + (size_t)row * L;
    const __nv_bfloat16* prow = P + (size_t)row * L;
    __nv_bfloat16* drow = dS + (size_t)row * L;
    const int n = causal ? t + 1 : L;
    float dot = 0.f;
    for (int s = lane; s < n; s += 32) dot = fmaf(__bfloat162float(prow[s]), grow[s], dot);
    dot = warp_sum(dot);
    for (int s = lane; s < L; s += 32)
        drow[s] = __float2bfloat16_rn(s < n ? __bfloat162float(prow[s]) * (grow[s] - dot) * scale : 0.f);
}

// The same gradient with the row held in registers (rows of at most NV * 128,
// read once with 16-byte loads of dP and 8-byte loads of P): lane l owns
// entries 4l .. 4l + 3 of every 128.  When causal, dS is written only up to
// the end of the row's 256-wide tile, as P is: the products that read dS
// (dS K up to the end of each row tile, dS^T Q from each row tile's diagonal
// on) never read further.
template <int NV>
__global__ void __launch_bounds__(kRowWarps * 32, NV <= 8 ? 3 : 1) sru_softmax_backward_rows_reg_kernel(
    const float* __restrict__ dP, const __nv_bfloat16* __restrict__ P, __nv_bfloat16* __restrict__ dS, int L, int rows,
    float scale, int causal) {
    const int row = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (row >= rows) return;
    const int t = row % L;
    const float4* grow = reinterpret_cast<const float4*>(dP + (size_t)row * L);
    const uint2* prow = reinterpret_cast<const uint2*>(P + (size_t)row * L);
    uint2* drow = reinterpret_cast<uint2*>(dS + (size_t)row * L);
    const int n = causal ? t + 1 : L;
    const int end = causal ? min(L, (t / 256 + 1) * 256) : L;  // written: [0, end)
    float4 gr[NV];
    uint2 pr[NV];  // 4 bf16
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int s0 = k * 128 + lane * 4;
        gr[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        pr[k] = make_uint2(0u, 0u);
        if (s0 < n) {
            gr[k] = grow[s0 / 4];
            pr[k] = prow[s0 / 4];
        }
    }
    // entry e of chunk k as fp32, 0 where invisible (s >= n)
    auto pval = [&](int k, int e) {
        const uint32_t w = e < 2 ? pr[k].x : pr[k].y;
        const float v = __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
        return k * 128 + lane * 4 + e < n ? v : 0.f;
    };
    auto gval = [&](int k, int e) {
        const float v = e == 0 ? gr[k].x : e == 1 ? gr[k].y : e == 2 ? gr[k].z : gr[k].w;
        return k * 128 + lane * 4 + e < n ? v : 0.f;
    };
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) dot = fmaf(pval(k, e), gval(k, e), dot);
    dot = warp_sum(dot);
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int s0 = k * 128 + lane * 4;
        if (s0 >= end) continue;
        // invisible entries have p = 0, so they come out as 0
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = pval(k, e) * (gval(k, e) - dot) * scale;
        __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(o[2], o[3]);
        drow[s0 / 4] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
}

// Gradient through R = Z (no norm) or R = layernorm(Z) gamma + beta, with
// Z = Q + alpha A recomputed exactly as the forward did.  Row m:
//   no norm:  dZ = dR
//   norm:     Zhat = (Z - mean) * rstd,  dZhat = dR * gamma,
//             dZ = rstd * (dZhat - mean(dZhat) - Zhat * mean(dZhat * Zhat))
// writes dQ = dZ (fp32; the attention and projection terms are added later)
// and dA = bf16(alpha dZ), and, with the norm, the row's mean and rstd (for
// the parameter gradients).
__global__ void __launch_bounds__(kRowWarps * 32) sru_norm_backward_kernel(
    const float* __restrict__ dR, const __nv_bfloat16* __restrict__ Q, const float* __restrict__ A, float alpha,
    const float* __restrict__ gamma, float* __restrict__ dQ, __nv_bfloat16* __restrict__ dA,
    float2* __restrict__ stats, int M, int dp) {
    const int m = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (m >= M) return;
    const float* dr = dR + (size_t)m * dp;
    float* dq = dQ + (size_t)m * dp;
    __nv_bfloat16* da = dA + (size_t)m * dp;
    if (gamma == nullptr) {
        for (int j = lane; j < dp; j += 32) {
            const float g = dr[j];
            dq[j] = g;
            da[j] = __float2bfloat16_rn(alpha * g);
        }
        return;
    }
    const __nv_bfloat16* q = Q + (size_t)m * dp;
    const float* a = A + (size_t)m * dp;
    float sum = 0.f;
    for (int j = lane; j < dp; j += 32) sum += fmaf(alpha, a[j], __bfloat162float(q[j]));
    const float mean = warp_sum(sum) / (float)dp;
    float sq = 0.f;
    for (int j = lane; j < dp; j += 32) {
        const float z = fmaf(alpha, a[j], __bfloat162float(q[j])) - mean;
        sq = fmaf(z, z, sq);
    }
    const float rstd = rsqrtf(warp_sum(sq) / (float)dp + kLayerNormEps);
    float s1 = 0.f, s2 = 0.f;
    for (int j = lane; j < dp; j += 32) {
        const float zh = (fmaf(alpha, a[j], __bfloat162float(q[j])) - mean) * rstd;
        const float g = dr[j] * gamma[j];
        s1 += g;
        s2 = fmaf(g, zh, s2);
    }
    s1 = warp_sum(s1) / (float)dp;
    s2 = warp_sum(s2) / (float)dp;
    for (int j = lane; j < dp; j += 32) {
        const float zh = (fmaf(alpha, a[j], __bfloat162float(q[j])) - mean) * rstd;
        const float g = dr[j] * gamma[j];
        const float dz = rstd * (g - s1 - zh * s2);
        dq[j] = dz;
        da[j] = __float2bfloat16_rn(alpha * dz);
    }
    if (lane == 0) stats[m] = make_float2(mean, rstd);
}

// The same gradient with the row held in registers (d' at most NV * 128, each
// input read once): lane l owns features 4l .. 4l + 3 of every 128.  The
// row's inputs are loaded first (NormRowIn), so that a caller walking several
// rows can have the next row's loads in flight while this one is computed.
template <int NV>
struct NormRowIn {
    float4 r[NV];  // dR
    float4 a[NV];  // A (with the norm)
    uint2 q[NV];   // Q, 4 bf16 (with the norm)
};
template <int NV>
__device__ __forceinline__ void load_norm_row(NormRowIn<NV>& in, const float* __restrict__ dR,
                                              const __nv_bfloat16* __restrict__ Q, const float* __restrict__ A,
                                              bool norm, int m, int dp, int lane) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int j0 = k * 128 + lane * 4;
        if (j0 >= dp) continue;
        in.r[k] = reinterpret_cast<const float4*>(dR + (size_t)m * dp)[j0 / 4];
        if (norm) {
            in.q[k] = reinterpret_cast<const uint2*>(Q + (size_t)m * dp)[j0 / 4];
            in.a[k] = reinterpret_cast<const float4*>(A + (size_t)m * dp)[j0 / 4];
        }
    }
}
// Row m's inputs as fp32: g = dR, z = Q + alpha A (with the norm); returns the
// lane's sum of z.  After this the NormRowIn may be reloaded.
template <int NV>
__device__ __forceinline__ float unpack_norm_row(const NormRowIn<NV>& in, float alpha, bool norm, int dp, int lane,
                                                 float (&g)[NV][4], float (&z)[NV][4]) {
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int j0 = k * 128 + lane * 4;
        if (j0 >= dp) {
#pragma unroll
            for (int e = 0; e < 4; ++e) g[k][e] = z[k][e] = 0.f;
            continue;
        }
        const float4 r4 = in.r[k];
        g[k][0] = r4.x;
        g[k][1] = r4.y;
        g[k][2] = r4.z;
        g[k][3] = r4.w;
        if (norm) {
            const uint2 qq = in.q[k];
            const float4 aa = in.a[k];
            const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qq.x));
            const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qq.y));
            z[k][0] = fmaf(alpha, aa.x, q01.x);
            z[k][1] = fmaf(alpha, aa.y, q01.y);
            z[k][2] = fmaf(alpha, aa.z, q23.x);
            z[k][3] = fmaf(alpha, aa.w, q23.y);
            sum += z[k][0] + z[k][1] + z[k][2] + z[k][3];
        }
    }
    return sum;
}
// Row m's gradient from its unpacked inputs.  With PARAMS (gamma given) row
// m's terms of the parameter gradients are added to the lane's running sums:
// pg += dR * Zhat (dgamma), pb += dR (dbeta).
template <int NV, bool PARAMS>
__device__ __forceinline__ void finish_norm_row(float (&g)[NV][4], float (&z)[NV][4], float sum, float alpha,
                                                const float* __restrict__ gamma, float* __restrict__ dQ,
                                                __nv_bfloat16* __restrict__ dA, float2* __restrict__ stats, int m,
                                                int dp, int lane, float (&pg)[NV][4], float (&pb)[NV][4]) {
    float4* dq = reinterpret_cast<float4*>(dQ + (size_t)m * dp);
    uint2* da = reinterpret_cast<uint2*>(dA + (size_t)m * dp);
    if (gamma != nullptr) {
        const float mean = warp_sum(sum) / (float)dp;
        float sq = 0.f;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            if (k * 128 + lane * 4 >= dp) continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) sq = fmaf(z[k][e] - mean, z[k][e] - mean, sq);
        }
        const float rstd = rsqrtf(warp_sum(sq) / (float)dp + kLayerNormEps);
        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            const int j0 = k * 128 + lane * 4;
            if (j0 >= dp) continue;
            const float4 g4 = *reinterpret_cast<const float4*>(gamma + j0);
            const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                z[k][e] = (z[k][e] - mean) * rstd;  // Zhat from here on
                if (PARAMS) {
                    pg[k][e] = fmaf(g[k][e], z[k][e], pg[k][e]);
                    pb[k][e] += g[k][e];
                }
                g[k][e] *= gv[e];  // dZhat = dR * gamma
                s1 += g[k][e];
                s2 = fmaf(g[k][e], z[k][e], s2);
            }
        }
        s1 = warp_sum(s1) / (float)dp;
        s2 = warp_sum(s2) / (float)dp;
#pragma unroll
        for (int k = 0; k < NV; ++k) {
            if (k * 128 + lane * 4 >= dp) continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) g[k][e] = rstd * (g[k][e] - s1 - z[k][e] * s2);
        }
        if (lane == 0) stats[m] = make_float2(mean, rstd);
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int j0 = k * 128 + lane * 4;
        if (j0 >= dp) continue;
        dq[j0 / 4] = make_float4(g[k][0], g[k][1], g[k][2], g[k][3]);
        __nv_bfloat162 lo = __floats2bfloat162_rn(alpha * g[k][0], alpha * g[k][1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(alpha * g[k][2], alpha * g[k][3]);
        da[j0 / 4] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
}

template <int NV>
__global__ void __launch_bounds__(kRowWarps * 32) sru_norm_backward_reg_kernel(
    const float* __restrict__ dR, const __nv_bfloat16* __restrict__ Q, const float* __restrict__ A, float alpha,
    const float* __restrict__ gamma, float* __restrict__ dQ, __nv_bfloat16* __restrict__ dA,
    float2* __restrict__ stats, int M, int dp) {
    const int m = blockIdx.x * kRowWarps + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (m >= M) return;
    NormRowIn<NV> in;
    load_norm_row<NV>(in, dR, Q, A, gamma != nullptr, m, dp, lane);
    float g[NV][4], z[NV][4];
    const float sum = unpack_norm_row<NV>(in, alpha, gamma != nullptr, dp, lane, g, z);
    float pg[NV][4], pb[NV][4];  // not used without PARAMS
    finish_norm_row<NV, false>(g, z, sum, alpha, gamma, dQ, dA, stats, m, dp, lane, pg, pb);
}

// The norm's parameter gradients, first stage: slice y of the rows (rows
// [y * kNormRows, (y + 1) * kNormRows)) summed per feature j in fp32, in row
// order, into part[y][0][j] (dgamma: dR * Zhat) and part[y][1][j] (dbeta: dR).
// This kernel re-reads dR, Q and A; sru_norm_backward_params_reg_kernel
// below does the same stage inside the norm's backward for d' <= 1024.
constexpr int kNormRows = 32;
constexpr int kNormParamThreads = 256;
__global__ void __launch_bounds__(kNormParamThreads) sru_norm_param_partial_kernel(
    const float* __restrict__ dR, const __nv_bfloat16* __restrict__ Q, const float* __restrict__ A, float alpha,
    const float2* __restrict__ stats, float* __restrict__ part, int M, int dp) {
    const int j = blockIdx.x * kNormParamThreads + threadIdx.x;
    if (j >= dp) return;
    const int m0 = blockIdx.y * kNormRows, m1 = min(M, m0 + kNormRows);
    float sg = 0.f, sb = 0.f;
    for (int m = m0; m < m1; ++m) {
        const size_t e = (size_t)m * dp + j;
        const float2 st = stats[m];
        const float zh = (fmaf(alpha, A[e], __bfloat162float(Q[e])) - st.x) * st.y;
        sg = fmaf(dR[e], zh, sg);
        sb += dR[e];
    }
    part[((size_t)blockIdx.y * 2 + 0) * dp + j] = sg;
    part[((size_t)blockIdx.y * 2 + 1) * dp + j] = sb;
}

// The norm's backward and the first stage of its parameter gradients in one
// pass (gamma given, d' at most NV * 128), on a grid that stays resident:
// warp w of CTA y takes rows (y + i * gridDim.x) * kRowWarps + w for i = 0,
// 1, ... (so every warp has the same number of rows, give or take one), keeps
// its sums of dR * Zhat and dR per feature in registers, and the warps' sums
// are added in warp order into slice y: part[y][0][j] (dgamma) and
// part[y][1][j] (dbeta).  For a given grid the order is fixed, so the result
// is the same on every run.
template <int NV>
__global__ void __launch_bounds__(kRowWarps * 32, NV <= 4 ? 2 : 1) sru_norm_backward_params_reg_kernel(
    const float* __restrict__ dR, const __nv_bfloat16* __restrict__ Q, const float* __restrict__ A, float alpha,
    const float* __restrict__ gamma, float* __restrict__ dQ, __nv_bfloat16* __restrict__ dA,
    float2* __restrict__ stats, float* __restrict__ part, int M, int dp) {
    __shared__ float red[2][NV * 128];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    float pg[NV][4], pb[NV][4];
#pragma unroll
    for (int k = 0; k < NV; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) pg[k][e] = pb[k][e] = 0.f;
    const int stride = gridDim.x * kRowWarps;
    // the next row's loads are issued as soon as this row's inputs are unpacked,
    // so they are in flight while this row is computed
    NormRowIn<NV> in;
    int m = blockIdx.x * kRowWarps + warp;
    if (m < M) load_norm_row<NV>(in, dR, Q, A, true, m, dp, lane);
#pragma unroll 1
    for (; m < M; m += stride) {
        float g[NV][4], z[NV][4];
        const float sum = unpack_norm_row<NV>(in, alpha, true, dp, lane, g, z);
        if (m + stride < M) load_norm_row<NV>(in, dR, Q, A, true, m + stride, dp, lane);
        finish_norm_row<NV, true>(g, z, sum, alpha, gamma, dQ, dA, stats, m, dp, lane, pg, pb);
    }
    for (int w = 0; w < kRowWarps; ++w) {
        if (warp == w) {
#pragma unroll
            for (int k = 0; k < NV; ++k) {
                const int j0 = k * 128 + lane * 4;
                if (j0 >= dp) continue;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    red[0][j0 + e] = w == 0 ? pg[k][e] : red[0][j0 + e] + pg[k][e];
                    red[1][j0 + e] = w == 0 ? pb[k][e] : red[1][j0 + e] + pb[k][e];
                }
            }
        }
        __syncthreads();
    }
    float* out = part + (size_t)blockIdx.x * 2 * dp;
    for (int c = threadIdx.x; c < 2 * dp; c += kRowWarps * 32) out[c] = red[c / dp][c % dp];
}

// Second stage: column c of the slices' partial sums (c < d': dgamma, else
// dbeta), in fp64.  A block owns kNormRedCols columns; its kNormRedGroups
// thread groups each sum slices g, g + kNormRedGroups, ... in increasing
// order, and the groups are then added in increasing order: a fixed order,
// so the result is the same on every run.
constexpr int kNormRedCols = 32, kNormRedGroups = 32;
__global__ void __launch_bounds__(kNormRedCols * kNormRedGroups) sru_norm_param_reduce_kernel(
    const float* __restrict__ part, int slices, int dp, float* __restrict__ dgamma, float* __restrict__ dbeta) {
    __shared__ double acc[kNormRedGroups][kNormRedCols];
    const int col = threadIdx.x % kNormRedCols, grp = threadIdx.x / kNormRedCols;
    const int c = blockIdx.x * kNormRedCols + col;
    double sum = 0.0;
    if (c < 2 * dp) {
#pragma unroll 4
        for (int y = grp; y < slices; y += kNormRedGroups) sum += (double)part[(size_t)y * 2 * dp + c];
    }
    acc[grp][col] = sum;
    __syncthreads();
    if (grp != 0 || c >= 2 * dp) return;
    double t = 0.0;
#pragma unroll
    for (int k = 0; k < kNormRedGroups; ++k) t += acc[k][col];
    if (c < dp)
        dgamma[c] = (float)t;
    else
        dbeta[c - dp] = (float)t;
}

// out[i] = bf16(a[i] + b[i]), four at a time (n a multiple of 4, all 16-byte aligned).
__global__ void __launch_bounds__(256) sru_add_to_bf16_kernel(const float4* __restrict__ a, const float4* __restrict__ b,
                                                              uint2* __restrict__ out, size_t n4) {
    for (size_t i = blockIdx.x * (size_t)256 + threadIdx.x; i < n4; i += (size_t)gridDim.x * 256) {
        const float4 u = a[i], v = b[i];
        __nv_bfloat162 lo = __floats2bfloat162_rn(u.x + v.x, u.y + v.y), hi = __floats2bfloat162_rn(u.z + v.z, u.w + v.w);
        out[i] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
}

}  // namespace sru
