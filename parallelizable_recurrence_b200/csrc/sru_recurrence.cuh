// sru_recurrence.cuh -- the element-wise SRU recurrence on sm_100a.
//
// Method: "When Attention Meets Fast Recurrence" (T. Lei), background section
// on SRU, Eqs. (2)-(5).  Once U is known every (direction, batch row b,
// channel j) stream is independent, so each thread owns one stream and walks
// t sequentially with the state c in a register.  A CTA owns CJ consecutive
// channels of one (b, direction); the U / x / dh tiles of T consecutive time
// steps are brought into shared memory by TMA (cp.async.bulk.tensor) through
// an S-stage mbarrier ring, so (S-1)*T steps of input are in flight while T
// steps are computed.  Outputs are written with coalesced stores (a warp
// writes 32 consecutive channels of one time step).
//
// The backward pass re-runs the forward over one chunk of T steps from the
// state checkpoint the forward stored at the chunk start (keeping c, f and r
// of the chunk in registers), then walks the chunk in reverse.  The partial
// sums of dv and db are accumulated per thread in double precision and
// reduced over the batch in a fixed order by a second kernel.
#pragma once

#include "sru_ptx.cuh"

namespace sru {

constexpr int kChunkT = 16;  // time steps per pipeline stage == checkpoint interval
constexpr int kRecCJ = 64;   // channels (threads) per CTA
constexpr int kFwdStages = 4;
constexpr int kBwdStages = 3;

// Per-channel constants of Eqs. (2)-(3), pre-scaled by -log2(e) so that one
// FMA gives the exponent of 2 in sigma(z) = 1 / (1 + 2^(-z log2 e)):
//   nvf = -v_f log2(e), nbf = -b_f log2(e)  (and the same for the reset gate).
struct GateParams {
    float vf, vr, bf, br;      // as given (the backward needs v_f, v_r)
    float nvf, nvr, nbf, nbr;  // scaled by -log2(e)
};
constexpr float kNegLog2e = -1.4426950408889634f;

__device__ __forceinline__ GateParams make_gate_params(float vf, float vr, float bf, float br) {
    GateParams p;
    p.vf = vf;
    p.vr = vr;
    p.bf = bf;
    p.br = br;
    p.nvf = __fmul_rn(vf, kNegLog2e);
    p.nvr = __fmul_rn(vr, kNegLog2e);
    p.nbf = __fmul_rn(bf, kNegLog2e);
    p.nbr = __fmul_rn(br, kNegLog2e);
    return p;
}

// 2^x and 1/x with the single-instruction approximations of the PTX ISA
// (ex2.approx: relative error ~2^-22; rcp.approx: within 1 ulp).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// logistic sigma(z) given e = -z log2(e): 1 / (1 + 2^e); saturates to exactly 0 and 1.
__device__ __forceinline__ float sigmoid_nl2(float e) { return rcp_approx(__fadd_rn(1.0f, ex2_approx(e))); }
// logistic sigma(u + b) for a gate with no peephole term (v = 0)
__device__ __forceinline__ float sigmoid_f(float z) { return sigmoid_nl2(__fmul_rn(z, kNegLog2e)); }

// One step of Eqs. (2)-(4): returns c[t] from c[t-1], and the gate values.
// Every operation is explicitly rounded so the forward and the backward's
// recomputation of a chunk produce bit-identical states.
__device__ __forceinline__ float sru_cell(float c, float uc, float uf, float ur, const GateParams& p,
                                          float& f, float& r) {
    f = sigmoid_nl2(__fmaf_rn(p.nvf, c, __fmaf_rn(uf, kNegLog2e, p.nbf)));
    r = sigmoid_nl2(__fmaf_rn(p.nvr, c, __fmaf_rn(ur, kNegLog2e, p.nbr)));
    return __fmaf_rn(f, __fsub_rn(c, uc), uc);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Bit i set: row t0+i of this chunk exists (t < L) and is not padded.  Whole warp calls.
__device__ __forceinline__ uint32_t chunk_valid_bits(const uint8_t* __restrict__ mask, int t0, int L, int B,
                                                     int b, int lane) {
    bool ok = lane < kChunkT && t0 + lane < L;
    if (ok && mask != nullptr) ok = mask[(size_t)(t0 + lane) * B + b] == 0;
    return __ballot_sync(0xffffffffu, ok);
}
__device__ __forceinline__ uint32_t chunk_inrange_bits(int t0, int L) {
    const int n = L - t0;
    return n >= kChunkT ? ((1u << kChunkT) - 1u) : ((1u << n) - 1u);
}

// After a failed wait: thread 0 waits (bounded) for the loads it issued that
// have not landed yet, so no copy is still writing this CTA's shared memory.
template <int S>
__device__ __forceinline__ void drain_pending_loads(uint64_t* full, uint32_t pending, uint32_t phase_bits) {
#pragma unroll
    for (int s = 0; s < S; ++s)
        if ((pending >> s) & 1u) mbar_wait(&full[s], (phase_bits >> s) & 1u, kErrTimeoutLoad);
}

// Eqs. (2)-(5) over one chunk of kChunkT rows staged in shared memory
// (us: [T][3][CJ] gate blocks, xs: [T][CJ]), walked in the direction's time
// order from state c.  Writes h for the rows that exist (0 at padded rows) and
// returns the state after the chunk.
template <typename UT>
__device__ __forceinline__ float fwd_chunk(const UT* __restrict__ us, const float* __restrict__ xs,
                                           uint32_t valid, uint32_t inrange, float c, const GateParams& p,
                                           float alpha, int dir, float* __restrict__ hp, size_t h_tstride,
                                           bool jok, int tid) {
    constexpr uint32_t kFull = (1u << kChunkT) - 1u;
    if (valid == kFull) {  // every row present and unpadded: no per-row predicates
        if (dir == 0) {
#pragma unroll
            for (int i = 0; i < kChunkT; ++i) {
                float f, r;
                c = sru_cell(c, to_f32(us[(i * 3 + 0) * kRecCJ + tid]), to_f32(us[(i * 3 + 1) * kRecCJ + tid]),
                             to_f32(us[(i * 3 + 2) * kRecCJ + tid]), p, f, r);
                const float ax = __fmul_rn(alpha, xs[i * kRecCJ + tid]);
                if (jok) hp[(size_t)i * h_tstride] = __fmaf_rn(r, __fsub_rn(c, ax), ax);  // Eq. (5)
            }
        } else {
#pragma unroll
            for (int i = kChunkT - 1; i >= 0; --i) {
                float f, r;
                c = sru_cell(c, to_f32(us[(i * 3 + 0) * kRecCJ + tid]), to_f32(us[(i * 3 + 1) * kRecCJ + tid]),
                             to_f32(us[(i * 3 + 2) * kRecCJ + tid]), p, f, r);
                const float ax = __fmul_rn(alpha, xs[i * kRecCJ + tid]);
                if (jok) hp[(size_t)i * h_tstride] = __fmaf_rn(r, __fsub_rn(c, ax), ax);
            }
        }
        return c;
    }
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = dir == 0 ? q : kChunkT - 1 - q;
        if (!((inrange >> i) & 1u)) continue;
        float hv = 0.f;
        if ((valid >> i) & 1u) {
            float f, r;
            c = sru_cell(c, to_f32(us[(i * 3 + 0) * kRecCJ + tid]), to_f32(us[(i * 3 + 1) * kRecCJ + tid]),
                         to_f32(us[(i * 3 + 2) * kRecCJ + tid]), p, f, r);
            const float ax = __fmul_rn(alpha, xs[i * kRecCJ + tid]);
            hv = __fmaf_rn(r, __fsub_rn(c, ax), ax);  // Eq. (5): r*c + (1-r)*alpha*x
        }
        if (jok) hp[(size_t)i * h_tstride] = hv;
    }
    return c;
}

template <typename UT>
struct FwdLayout {
    static constexpr int U_BYTES = kChunkT * 3 * kRecCJ * (int)sizeof(UT);
    static constexpr int X_BYTES = kChunkT * kRecCJ * 4;
    static constexpr int STAGE = U_BYTES + X_BYTES;
    static constexpr int BAR_OFF = kFwdStages * STAGE;
    static constexpr int SMEM = BAR_OFF + 64 + 128;  // barriers + alignment slack
};

// Forward.  Grid (ceil(d/CJ), B, n_dir), block CJ threads.
//   map_u: 4-D (d, 3, B*n_dir, L) of UT, box (CJ, 3, 1, T)
//   map_x: 3-D (d, B, L) fp32, box (CJ, 1, T)
template <typename UT>
__global__ void __launch_bounds__(kRecCJ) sru_fwd_seq_kernel(
    const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_x,
    const float* __restrict__ v, const float* __restrict__ bias, const float* __restrict__ c0,
    const uint8_t* __restrict__ mask, float* __restrict__ h, float* __restrict__ c_T, float* __restrict__ ckpt,
    int L, int B, int d, int n_dir, float alpha) {
    using Lay = FwdLayout<UT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);

    const int tid = threadIdx.x, lane = tid & 31;
    const int j0 = blockIdx.x * kRecCJ, j = j0 + tid;
    const int b = blockIdx.y, dir = blockIdx.z;
    const int bd = b * n_dir + dir;
    const bool jok = j < d;
    const int nch = (L + kChunkT - 1) / kChunkT;

    GateParams p = make_gate_params(0.f, 0.f, 0.f, 0.f);
    float c = 0.f;
    if (jok) {
        p = make_gate_params(v[(dir * 2 + 0) * d + j], v[(dir * 2 + 1) * d + j], bias[(dir * 2 + 0) * d + j],
                             bias[(dir * 2 + 1) * d + j]);
        if (c0 != nullptr) c = c0[(size_t)bd * d + j];
    }
    if (tid == 0) {
        for (int s = 0; s < kFwdStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_u);
        tma_prefetch_desc(&map_x);
    }
    __syncthreads();

    auto time_chunk = [&](int k) { return dir == 0 ? k : nch - 1 - k; };
    uint32_t pending = 0;  // thread 0: stages with a load in flight
    // warp 0 issues the loads of processing chunk k into stage k % S (skipped if fully padded)
    auto issue = [&](int k) {
        const int t0 = time_chunk(k) * kChunkT;
        const uint32_t valid = chunk_valid_bits(mask, t0, L, B, b, lane);
        if (lane == 0 && valid != 0u) {
            const int s = k % kFwdStages;
            pending |= 1u << s;
            uint8_t* st = smem + s * Lay::STAGE;
            mbar_arrive_expect_tx(&full[s], Lay::STAGE);
            tma_load_4d(st, &map_u, &full[s], j0, 0, bd, t0);
            tma_load_3d(st + Lay::U_BYTES, &map_x, &full[s], j0, b, t0);
        }
    };
    if (tid < 32)
        for (int k = 0; k < kFwdStages && k < nch; ++k) issue(k);

    uint32_t phase_bits = 0;
    const size_t h_tstride = (size_t)B * n_dir * d;
    for (int k = 0; k < nch; ++k) {
        const int s = k % kFwdStages;
        const int tc = time_chunk(k), t0 = tc * kChunkT;
        const uint32_t valid = chunk_valid_bits(mask, t0, L, B, b, lane);
        const uint32_t inrange = chunk_inrange_bits(t0, L);
        if (ckpt != nullptr && jok) ckpt[((size_t)tc * B * n_dir + bd) * d + j] = c;
        if (valid != 0u) {
            const bool ok = mbar_wait(&full[s], (phase_bits >> s) & 1u, kErrTimeoutLoad);
            if (__syncthreads_or(!ok)) {  // a load never landed: give up (error recorded)
                if (tid == 0) drain_pending_loads<kFwdStages>(full, pending, phase_bits);
                return;
            }
            phase_bits ^= 1u << s;
            pending &= ~(1u << s);
        }
        const UT* us = reinterpret_cast<const UT*>(smem + s * Lay::STAGE);
        const float* xs = reinterpret_cast<const float*>(smem + s * Lay::STAGE + Lay::U_BYTES);
        float* hp = h + (size_t)t0 * h_tstride + (size_t)bd * d + j;
        c = fwd_chunk<UT>(us, xs, valid, inrange, c, p, alpha, dir, hp, h_tstride, jok, tid);
        __syncthreads();  // every thread is done with stage s
        if (tid < 32 && k + kFwdStages < nch) issue(k + kFwdStages);
    }
    if (jok) c_T[(size_t)bd * d + j] = c;
}

// Backward over one chunk staged in shared memory (us, xs, dhs and, with
// ACC_DX, the other direction's dx in dxin), given the state c entering the
// chunk in forward order and the state gradient g leaving it.  Re-runs the
// forward over the chunk keeping c, f and r in registers, then walks it in
// reverse: writes dU and dx for the rows that exist, accumulates the dv/db
// partial sums in acc = {dv_f, dv_r, db_f, db_r}, and updates g.
template <typename UT, typename DUT, bool ACC_DX, int DIR>
__device__ __forceinline__ void bwd_chunk(const UT* __restrict__ us, const float* __restrict__ xs,
                                          const float* __restrict__ dhs, const float* __restrict__ dxin,
                                          uint32_t valid, uint32_t inrange, float c, const GateParams& p,
                                          float alpha, float& g, double (&acc)[4], DUT* __restrict__ dUp,
                                          float* __restrict__ dxp, size_t u_tstride, size_t x_tstride, int d,
                                          bool jok, int tid) {
    constexpr uint32_t kFull = (1u << kChunkT) - 1u;
    const bool full = valid == kFull;
    float cp[kChunkT], fs[kChunkT], rs[kChunkT];
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = DIR == 0 ? q : kChunkT - 1 - q;
        cp[i] = c;
        fs[i] = 0.f;
        rs[i] = 0.f;
        if (full || ((valid >> i) & 1u))
            c = sru_cell(c, to_f32(us[(i * 3 + 0) * kRecCJ + tid]), to_f32(us[(i * 3 + 1) * kRecCJ + tid]),
                         to_f32(us[(i * 3 + 2) * kRecCJ + tid]), p, fs[i], rs[i]);
    }
    // chunk partial sums in fp32 (16 terms), folded into the double totals once per chunk
    float s_vf = 0.f, s_vr = 0.f, s_bf = 0.f, s_br = 0.f;
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = DIR == 0 ? kChunkT - 1 - q : q;
        if (!full && !((inrange >> i) & 1u)) continue;
        float duc = 0.f, dzf = 0.f, dzr = 0.f, dxv = 0.f;
        const bool row = full || ((valid >> i) & 1u);
        if (row) {
            const float f = fs[i], r = rs[i], cpv = cp[i];
            const float uc = to_f32(us[(i * 3 + 0) * kRecCJ + tid]);
            const float ax = __fmul_rn(alpha, xs[i * kRecCJ + tid]);
            const float dhv = dhs[i * kRecCJ + tid];
            const float cn = __fmaf_rn(f, __fsub_rn(cpv, uc), uc);
            const float G = __fmaf_rn(dhv, r, g);  // dLoss/dc[t]
            const float omr = __fsub_rn(1.f, r), omf = __fsub_rn(1.f, f);
            dxv = __fmul_rn(__fmul_rn(dhv, omr), alpha);
            dzf = __fmul_rn(__fmul_rn(G, __fsub_rn(cpv, uc)), __fmul_rn(f, omf));
            dzr = __fmul_rn(__fmul_rn(dhv, __fsub_rn(cn, ax)), __fmul_rn(r, omr));
            duc = __fmul_rn(G, omf);
            g = __fmaf_rn(dzr, p.vr, __fmaf_rn(dzf, p.vf, __fmul_rn(G, f)));  // dLoss/dc[t-1]
            s_vf = __fmaf_rn(dzf, cpv, s_vf);
            s_vr = __fmaf_rn(dzr, cpv, s_vr);
            s_bf = __fadd_rn(s_bf, dzf);
            s_br = __fadd_rn(s_br, dzr);
        }
        if (jok) {
            dUp[(size_t)i * u_tstride] = from_f32<DUT>(duc);
            dUp[(size_t)i * u_tstride + d] = from_f32<DUT>(dzf);
            dUp[(size_t)i * u_tstride + 2 * d] = from_f32<DUT>(dzr);
            if (ACC_DX) {
                if (row) dxp[(size_t)i * x_tstride] = __fadd_rn(dxin[i * kRecCJ + tid], dxv);
            } else {
                dxp[(size_t)i * x_tstride] = dxv;
            }
        }
    }
    acc[0] += (double)s_vf;
    acc[1] += (double)s_vr;
    acc[2] += (double)s_bf;
    acc[3] += (double)s_br;
}

// A chunk with no valid row: zero dU (and dx unless accumulating); g passes through.
template <typename DUT, bool ACC_DX>
__device__ __forceinline__ void bwd_chunk_padded(uint32_t inrange, DUT* __restrict__ dUp, float* __restrict__ dxp,
                                                 size_t u_tstride, size_t x_tstride, int d, bool jok) {
    if (!jok) return;
#pragma unroll
    for (int i = 0; i < kChunkT; ++i) {
        if (!((inrange >> i) & 1u)) continue;
        dUp[(size_t)i * u_tstride] = from_f32<DUT>(0.f);
        dUp[(size_t)i * u_tstride + d] = from_f32<DUT>(0.f);
        dUp[(size_t)i * u_tstride + 2 * d] = from_f32<DUT>(0.f);
        if (!ACC_DX) dxp[(size_t)i * x_tstride] = 0.f;
    }
}

template <typename UT, bool ACC_DX>
struct BwdLayout {
    static constexpr int U_BYTES = kChunkT * 3 * kRecCJ * (int)sizeof(UT);
    static constexpr int V_BYTES = kChunkT * kRecCJ * 4;  // one fp32 (T, CJ) tile
    static constexpr int STAGE = U_BYTES + V_BYTES * (ACC_DX ? 3 : 2);
    static constexpr int BAR_OFF = kBwdStages * STAGE;
    static constexpr int SMEM = BAR_OFF + 64 + 128;
};

// Backward of direction DIR.  Grid (ceil(d/CJ), B), block CJ threads.
// ACC_DX: dx += this direction's highway gradient (dx already holds the other
// direction's, written by an earlier launch on the same stream), else dx = it.
//   map_dh: 3-D (d, B*n_dir, L) fp32; map_dxin: like map_x but over dx.
// DIR is a template parameter so the per-chunk register arrays are indexed
// with compile-time constants.
template <typename UT, typename DUT, bool ACC_DX, int DIR>
__global__ void __launch_bounds__(kRecCJ) sru_bwd_seq_kernel(
    const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_x,
    const __grid_constant__ CUtensorMap map_dh, const __grid_constant__ CUtensorMap map_dxin,
    const float* __restrict__ v, const float* __restrict__ bias, const uint8_t* __restrict__ mask,
    const float* __restrict__ ckpt, const float* __restrict__ dc_T, DUT* __restrict__ dU,
    float* __restrict__ dx, double* __restrict__ partial, float* __restrict__ dc0, int L, int B, int d,
    int n_dir, float alpha) {
    using Lay = BwdLayout<UT, ACC_DX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);

    const int tid = threadIdx.x, lane = tid & 31;
    const int j0 = blockIdx.x * kRecCJ, j = j0 + tid;
    constexpr int dir = DIR;
    const int b = blockIdx.y;
    const int bd = b * n_dir + dir;
    const bool jok = j < d;
    const int nch = (L + kChunkT - 1) / kChunkT;

    GateParams p = make_gate_params(0.f, 0.f, 0.f, 0.f);
    float g = 0.f;
    if (jok) {
        p = make_gate_params(v[(dir * 2 + 0) * d + j], v[(dir * 2 + 1) * d + j], bias[(dir * 2 + 0) * d + j],
                             bias[(dir * 2 + 1) * d + j]);
        if (dc_T != nullptr) g = dc_T[(size_t)bd * d + j];
    }
    if (tid == 0) {
        for (int s = 0; s < kBwdStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_u);
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_dh);
        if (ACC_DX) tma_prefetch_desc(&map_dxin);
    }
    __syncthreads();

    // backward processing chunk k covers time chunk: dir 0 walks time chunks downwards
    auto time_chunk = [&](int k) { return dir == 0 ? nch - 1 - k : k; };
    uint32_t pending = 0;  // thread 0: stages with a load in flight
    auto issue = [&](int k) {
        const int t0 = time_chunk(k) * kChunkT;
        const uint32_t valid = chunk_valid_bits(mask, t0, L, B, b, lane);
        if (lane == 0 && valid != 0u) {
            const int s = k % kBwdStages;
            pending |= 1u << s;
            uint8_t* st = smem + s * Lay::STAGE;
            mbar_arrive_expect_tx(&full[s], Lay::STAGE);
            tma_load_4d(st, &map_u, &full[s], j0, 0, bd, t0);
            tma_load_3d(st + Lay::U_BYTES, &map_x, &full[s], j0, b, t0);
            tma_load_3d(st + Lay::U_BYTES + Lay::V_BYTES, &map_dh, &full[s], j0, bd, t0);
            if (ACC_DX) tma_load_3d(st + Lay::U_BYTES + 2 * Lay::V_BYTES, &map_dxin, &full[s], j0, b, t0);
        }
    };
    if (tid < 32)
        for (int k = 0; k < kBwdStages && k < nch; ++k) issue(k);

    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    uint32_t phase_bits = 0;
    const size_t u_tstride = (size_t)B * n_dir * 3 * d;
    const size_t x_tstride = (size_t)B * d;
    for (int k = 0; k < nch; ++k) {
        const int s = k % kBwdStages;
        const int tc = time_chunk(k), t0 = tc * kChunkT;
        const uint32_t valid = chunk_valid_bits(mask, t0, L, B, b, lane);
        const uint32_t inrange = chunk_inrange_bits(t0, L);
        DUT* dUp = dU + (size_t)t0 * u_tstride + (size_t)bd * 3 * d + j;
        float* dxp = dx + (size_t)t0 * x_tstride + (size_t)b * d + j;
        if (valid == 0u) {
            bwd_chunk_padded<DUT, ACC_DX>(inrange, dUp, dxp, u_tstride, x_tstride, d, jok);
            __syncthreads();
            if (tid < 32 && k + kBwdStages < nch) issue(k + kBwdStages);
            continue;
        }
        const bool ok = mbar_wait(&full[s], (phase_bits >> s) & 1u, kErrTimeoutLoad);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) drain_pending_loads<kBwdStages>(full, pending, phase_bits);
            return;
        }
        phase_bits ^= 1u << s;
        pending &= ~(1u << s);

        const UT* us = reinterpret_cast<const UT*>(smem + s * Lay::STAGE);
        const float* xs = reinterpret_cast<const float*>(smem + s * Lay::STAGE + Lay::U_BYTES);
        const float* dhs = xs + kChunkT * kRecCJ;
        const float* dxin = dhs + kChunkT * kRecCJ;
        const float c_start = jok ? ckpt[((size_t)tc * B * n_dir + bd) * d + j] : 0.f;
        bwd_chunk<UT, DUT, ACC_DX, DIR>(us, xs, dhs, dxin, valid, inrange, c_start, p, alpha, g, acc, dUp, dxp,
                                        u_tstride, x_tstride, d, jok, tid);
        __syncthreads();
        if (tid < 32 && k + kBwdStages < nch) issue(k + kBwdStages);
    }
    if (jok) {
        dc0[(size_t)bd * d + j] = g;
        double* pp = partial + (size_t)bd * 4 * d + j;
        pp[0] = acc[0];
        pp[(size_t)d] = acc[1];
        pp[(size_t)2 * d] = acc[2];
        pp[(size_t)3 * d] = acc[3];
    }
}

// dv, db = sum over b of the per-row partial sums, in increasing b (deterministic).
// partial: (B, n_dir, 4, d) doubles, rows [dv_f, dv_r, db_f, db_r].
__global__ void sru_reduce_dvdb_kernel(const double* __restrict__ partial, int B, int d, int n_dir,
                                       float* __restrict__ dv, float* __restrict__ db) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= n_dir * 4 * d) return;
    const int dir = idx / (4 * d), q = (idx / d) % 4, j = idx % d;
    double s = 0.0;
    for (int bb = 0; bb < B; ++bb) s += partial[(((size_t)bb * n_dir + dir) * 4 + q) * d + j];
    if (q < 2)
        dv[(dir * 2 + q) * d + j] = (float)s;
    else
        db[(dir * 2 + q - 2) * d + j] = (float)s;
}

// L == 0: the final state is the initial state.
__global__ void sru_copy_state_kernel(const float* __restrict__ c0, float* __restrict__ out, size_t n) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = c0 != nullptr ? c0[i] : 0.f;
}

__global__ void sru_fill_f32_kernel(float* __restrict__ out, size_t n, float value) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = value;
}

}  // namespace sru
