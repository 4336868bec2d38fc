// sru_recurrence.cuh -- the element-wise SRU recurrence on sm_100a.
//
// Method: "When Attention Meets Fast Recurrence" (T. Lei), background section
// on SRU, Eqs. (2)-(5).  Once U is known every (direction, batch row b,
// channel j) stream is independent; each is walked sequentially over t with
// its state c in a register.
//
// Layout of the work: a CTA owns CJ (64; a build knob allows 32) consecutive channels of
// one (b, direction), CJ/2 threads; each thread owns two adjacent channels and
// advances both with the packed fp32x2 instructions of sm_100 (__ffma2_rn,
// __fadd2_rn, __fmul2_rn), so the two independent recurrences interleave and
// most arithmetic costs one instruction per pair.  The U / x / dh tiles of
// kChunkT consecutive steps are brought into shared memory by TMA
// (cp.async.bulk.tensor) through an S-stage mbarrier ring, so (S-1)*kChunkT
// steps of input are in flight while kChunkT steps are computed.  Outputs are
// written with coalesced 8-byte (fp32 pair) / 4-byte (bf16 pair) stores, or,
// for full chunks where it pays, over the chunk's input tile in shared memory
// and out by TMA stores (see the kernels).
//
// The backward re-runs the forward over one chunk from the state checkpoint
// the forward stored at the chunk start (keeping c, f and r of the chunk in
// registers), then walks it in reverse.  dv/db partial sums are fp32 within a
// chunk, fp64 per thread, and reduced over the batch in a fixed order.
#pragma once

#include "sru_ptx.cuh"

namespace sru {

constexpr int kChunkT = 16;          // time steps per pipeline stage == checkpoint interval
constexpr int kRecCJ = 64;           // channels per CTA
constexpr int kRecThreads = 32;      // one warp; thread i owns channels 2i and 2i+1 of the tile
// TMA ring depth of the sequential kernels: a template parameter S, from 2 up
// to these maxima, picked per launch so that the grid needs as few waves of
// resident CTAs as possible (each CTA walks the whole sequence, so a second,
// partly filled wave costs as much as the first).
constexpr int kFwdStages = 4;
constexpr int kBwdStages = 3;
constexpr float kNegLog2e = -1.4426950408889634f;

// ------------------------------------------------------------ scalar helpers
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

// -------------------------------------------------------------- pair helpers
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
// a - b, rounded once (the fma of -1*b + a is exact before its single rounding)
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, f2(-1.0f), a); }
__device__ __forceinline__ float2 sigmoid2_nl2(float2 e) {
    const float2 t = add2(f2(1.0f), make_float2(ex2_approx(e.x), ex2_approx(e.y)));
    return make_float2(rcp_approx(t.x), rcp_approx(t.y));
}

// Per-channel-pair constants of Eqs. (2)-(3), pre-scaled by -log2(e) so that
// one FMA gives the exponent of 2 in sigma(z) = 1 / (1 + 2^(-z log2 e)).
struct GateParams2 {
    float2 vf, vr;              // as given (the backward needs v_f, v_r)
    float2 nvf, nvr, nbf, nbr;  // -v log2(e), -b log2(e)
};
__device__ __forceinline__ GateParams2 make_gate_params2(float2 vf, float2 vr, float2 bf, float2 br) {
    GateParams2 p;
    p.vf = vf;
    p.vr = vr;
    p.nvf = mul2(vf, f2(kNegLog2e));
    p.nvr = mul2(vr, f2(kNegLog2e));
    p.nbf = mul2(bf, f2(kNegLog2e));
    p.nbr = mul2(br, f2(kNegLog2e));
    return p;
}

// One step of Eqs. (2)-(4) for two channels: returns c[t] from c[t-1] and the
// gate values.  Every operation is explicitly rounded, so the forward and the
// backward's recomputation of a chunk give bit-identical states.
__device__ __forceinline__ float2 sru_cell2(float2 c, float2 uc, float2 uf, float2 ur, const GateParams2& p,
                                            float2& f, float2& r) {
    f = sigmoid2_nl2(fma2(p.nvf, c, fma2(uf, f2(kNegLog2e), p.nbf)));
    r = sigmoid2_nl2(fma2(p.nvr, c, fma2(ur, f2(kNegLog2e), p.nbr)));
    return fma2(f, sub2(c, uc), uc);
}

// The two halves of sru_cell2, for chunks walked in two passes: the state
// chain needs only the forget gate (Eqs. (2), (4)); the reset gate (Eq. (3))
// and h (Eq. (5)) of every step of a chunk can then be computed without a
// dependency between steps.  Same operations as sru_cell2, so the same bits.
__device__ __forceinline__ float2 sru_forget2(float2 c, float2 uf, const GateParams2& p) {
    return sigmoid2_nl2(fma2(p.nvf, c, fma2(uf, f2(kNegLog2e), p.nbf)));
}
__device__ __forceinline__ float2 sru_reset2(float2 c, float2 ur, const GateParams2& p) {
    return sigmoid2_nl2(fma2(p.nvr, c, fma2(ur, f2(kNegLog2e), p.nbr)));
}

// Loads/stores of a channel pair (2 adjacent elements, 4- or 8-byte aligned).
__device__ __forceinline__ float2 load_pair(const __nv_bfloat16* p) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ float2 load_pair(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ void store_pair(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void store_pair(__nv_bfloat16* p, float2 v) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}
// p[0..1] += v with one 8-byte atomic (sm_90+ vector atomicAdd): used where
// exactly one addend arrives per element, so the result does not depend on
// timing.
__device__ __forceinline__ void add_pair(float* p, float2 v) { atomicAdd(reinterpret_cast<float2*>(p), v); }

// A channel pair of U as held in registers before use: the raw bf16x2 word
// (one 32-bit register) or the fp32 pair.
template <typename UT>
struct PairWord;
template <>
struct PairWord<__nv_bfloat16> {
    using T = uint32_t;
    static __device__ __forceinline__ T load(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }
    static __device__ __forceinline__ float2 unpack(T w) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
};
template <>
struct PairWord<float> {
    using T = float2;
    static __device__ __forceinline__ T load(const float* p) { return *reinterpret_cast<const float2*>(p); }
    static __device__ __forceinline__ float2 unpack(T w) { return w; }
};

// Lane i's row of the chunk starting at t0 (lanes below kChunkT): it exists
// (t < L) and is not padded.
__device__ __forceinline__ bool chunk_row_ok(const uint8_t* __restrict__ mask, int t0, int L, int B, int b,
                                             int lane) {
    bool ok = lane < kChunkT && t0 + lane < L;
    if (ok && mask != nullptr) ok = mask[(size_t)(t0 + lane) * B + b] == 0;
    return ok;
}
// The warp's vote on chunk_row_ok: bit i set for row t0+i.  CTAs of fewer than
// 32 threads (at least kChunkT) vote with their own lanes.
__device__ __forceinline__ uint32_t chunk_vote(bool ok) {
    const unsigned lanes = blockDim.x >= 32 ? 0xffffffffu : ((1u << blockDim.x) - 1u);
    return __ballot_sync(lanes, ok);
}
// Bit i set: row t0+i of this chunk exists (t < L) and is not padded.  Every
// thread of the warp (or of a CTA smaller than a warp) calls.
__device__ __forceinline__ uint32_t chunk_valid_bits(const uint8_t* __restrict__ mask, int t0, int L, int B,
                                                     int b, int lane) {
    return chunk_vote(chunk_row_ok(mask, t0, L, B, b, lane));
}
__device__ __forceinline__ uint32_t chunk_inrange_bits(int t0, int L) {
    const int n = L - t0;
    return n >= kChunkT ? ((1u << kChunkT) - 1u) : ((1u << n) - 1u);
}

// After a failed wait: lane 0 waits (bounded) for the loads it issued that
// have not landed yet, so no copy is still writing this CTA's shared memory.
template <int S>
__device__ __forceinline__ void drain_pending_loads(uint64_t* full, uint32_t pending, uint32_t phase_bits) {
#pragma unroll
    for (int s = 0; s < S; ++s)
        if ((pending >> s) & 1u) mbar_wait(&full[s], (phase_bits >> s) & 1u, kErrTimeoutLoad);
}

// ---------------------------------------------------------------- forward
// Eqs. (2)-(5) over one chunk of kChunkT rows staged in shared memory
// (us: [T][3][CJ] gate blocks, xs: [T][CJ]), walked in the direction's time
// order from state c, for this thread's channel pair (offset cj in the tile).
// Writes h for the rows that exist (0 at padded rows); returns the state.
// Fast path of fwd_chunk for a chunk whose 16 rows all exist and are valid,
// in direction DIR's time order: the chunk's operands are first copied from
// shared memory into registers, the 16 dependent steps then run on registers
// only, and the outputs are stored last.  With about one warp per SM
// sub-partition the serial chain of a step (two MUFU round trips) must not
// also wait on shared-memory loads or store addressing.
// STAGE: h is written over this thread's own x values in the chunk's
// shared-memory stage (copied to registers first) for the caller to store
// with TMA, instead of to global memory.
template <typename UT, int CJ, int DIR, bool STAGE = false>
__device__ __forceinline__ float2 fwd_chunk_full(const UT* __restrict__ us, const float* __restrict__ xs, float2 c,
                                                 const GateParams2& p, float2 alpha, float* __restrict__ hp,
                                                 size_t h_tstride, bool jok, int cj) {
    using PW = PairWord<UT>;
    typename PW::T wc[kChunkT], wf[kChunkT], wr[kChunkT];
    float2 wx[kChunkT];
#pragma unroll
    for (int i = 0; i < kChunkT; ++i) {
        wc[i] = PW::load(us + (i * 3 + 0) * CJ + cj);
        wf[i] = PW::load(us + (i * 3 + 1) * CJ + cj);
        wr[i] = PW::load(us + (i * 3 + 2) * CJ + cj);
        wx[i] = load_pair(xs + i * CJ + cj);
    }
    // pass 1: the state chain (forget gate and c only)
    float2 cprev[kChunkT], cs[kChunkT];
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = DIR == 0 ? q : kChunkT - 1 - q;
        cprev[i] = c;
        const float2 uc = PW::unpack(wc[i]);
        c = fma2(sru_forget2(c, PW::unpack(wf[i]), p), sub2(c, uc), uc);  // Eq. (4)
        cs[i] = c;
    }
    // pass 2: reset gate and h of every step, independent of one another
    float2 hv[kChunkT];
#pragma unroll
    for (int i = 0; i < kChunkT; ++i) {
        const float2 r = sru_reset2(cprev[i], PW::unpack(wr[i]), p);
        const float2 ax = mul2(alpha, wx[i]);
        hv[i] = fma2(r, sub2(cs[i], ax), ax);  // Eq. (5)
    }
    if (STAGE) {
        asm volatile("" ::: "memory");  // the x reads above precede the writes over them
#pragma unroll
        for (int i = 0; i < kChunkT; ++i) store_pair(const_cast<float*>(xs) + i * CJ + cj, hv[i]);
    } else if (jok) {
#pragma unroll
        for (int i = 0; i < kChunkT; ++i) store_pair(hp + (size_t)i * h_tstride, hv[i]);
    }
    return c;
}

template <typename UT, int CJ = kRecCJ, bool STAGE = false>
__device__ __forceinline__ float2 fwd_chunk(const UT* __restrict__ us, const float* __restrict__ xs,
                                            uint32_t valid, uint32_t inrange, float2 c, const GateParams2& p,
                                            float2 alpha, int dir, float* __restrict__ hp, size_t h_tstride,
                                            bool jok, int cj) {
    constexpr uint32_t kFull = (1u << kChunkT) - 1u;
    // (with STAGE, only full chunks come here)
    if (valid == kFull)
        return dir == 0 ? fwd_chunk_full<UT, CJ, 0, STAGE>(us, xs, c, p, alpha, hp, h_tstride, jok, cj)
                        : fwd_chunk_full<UT, CJ, 1, STAGE>(us, xs, c, p, alpha, hp, h_tstride, jok, cj);
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = dir == 0 ? q : kChunkT - 1 - q;
        if (!((inrange >> i) & 1u)) continue;
        float2 hv = f2(0.f);
        if ((valid >> i) & 1u) {
            float2 f, r;
            c = sru_cell2(c, load_pair(us + (i * 3 + 0) * CJ + cj), load_pair(us + (i * 3 + 1) * CJ + cj),
                          load_pair(us + (i * 3 + 2) * CJ + cj), p, f, r);
            const float2 ax = mul2(alpha, load_pair(xs + i * CJ + cj));
            hv = fma2(r, sub2(c, ax), ax);  // Eq. (5): r*c + (1-r)*alpha*x
        }
        if (jok) store_pair(hp + (size_t)i * h_tstride, hv);
    }
    return c;
}

template <typename UT, int CJ = kRecCJ, int S = kFwdStages>
struct FwdLayout {
    static constexpr int U_BYTES = kChunkT * 3 * CJ * (int)sizeof(UT);
    static constexpr int X_BYTES = kChunkT * CJ * 4;
    static constexpr int STAGE = U_BYTES + X_BYTES;
    static constexpr int BAR_OFF = S * STAGE;
    static constexpr int SMEM = BAR_OFF + 64 + 128;  // barriers + alignment slack
};

// Forward.  Grid (ceil(d/CJ), B, n_dir), CJ/2 threads (CJ/64 warps) per CTA.
//   map_u: 4-D (d, 3, B*n_dir, L) of UT, box (CJ, 3, 1, T)
//   map_x: 3-D (d, B, L) fp32, box (CJ, 1, T)
template <typename UT, int CJ, int S, bool STAGE_H = false>
__global__ void __launch_bounds__(CJ / 2) sru_fwd_seq_kernel(
    const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_x,
    const __grid_constant__ CUtensorMap map_h, const float* __restrict__ v, const float* __restrict__ bias,
    const float* __restrict__ c0, const uint8_t* __restrict__ mask, float* __restrict__ h, float* __restrict__ c_T,
    float* __restrict__ ckpt, const int* __restrict__ order, int L, int B, int d, int n_dir, float alpha) {
    using Lay = FwdLayout<UT, CJ, S>;
    // STAGE_H: full chunks leave through a TMA store of h written over the
    // stage's x tile; a stage is refilled one iteration after its store was
    // issued, so loads run S - 1 chunks ahead (rings of 3 or more stages).
    // Measured on B200 it pays only where the per-thread h stores throttle a
    // dense grid (L1024 B16 d3072: 138 -> 128 us) and costs elsewhere
    // (L1024 B16 d2048: 94 -> 105 us), so the host chooses per launch.
    constexpr bool kStage = STAGE_H && S >= 3;
    constexpr int kAhead = kStage ? S - 1 : S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);

    const int tid = threadIdx.x, lane = tid & 31, cj = 2 * tid;
    const int j0 = blockIdx.x * CJ, j = j0 + cj;
    // grid (d tiles, B, n_dir), or with `order` (d tiles, B * n_dir): the
    // (batch row, direction) streams longest first (padded layers)
    const int bd = order != nullptr ? order[blockIdx.y] : (int)(blockIdx.y * n_dir + blockIdx.z);
    const int b = bd / n_dir, dir = bd % n_dir;
    const bool jok = j < d;  // d is even, so the pair is either in or out
    const int nch = (L + kChunkT - 1) / kChunkT;

    GateParams2 p = make_gate_params2(f2(0.f), f2(0.f), f2(0.f), f2(0.f));
    float2 c = f2(0.f);
    if (jok) {
        p = make_gate_params2(load_pair(v + (dir * 2 + 0) * d + j), load_pair(v + (dir * 2 + 1) * d + j),
                              load_pair(bias + (dir * 2 + 0) * d + j), load_pair(bias + (dir * 2 + 1) * d + j));
        if (c0 != nullptr) c = load_pair(c0 + (size_t)bd * d + j);
    }
    const float2 alpha2 = f2(alpha);
    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_u);
        tma_prefetch_desc(&map_x);
        if (kStage) tma_prefetch_desc(&map_h);
    }
    __syncthreads();

    auto time_chunk = [&](int k) { return dir == 0 ? k : nch - 1 - k; };
    // the row-validity words of processing chunks k .. k + kAhead, slot k & 3: each is
    // voted on when its chunk's loads are issued, from mask bytes fetched one chunk
    // earlier, so no mask read sits on the chain
    uint32_t* vring = reinterpret_cast<uint32_t*>(full + S);
    uint32_t pending = 0;  // thread 0: stages with a load in flight
    // warp 0 issues the loads of processing chunk k into stage k % S (skipped if fully padded)
    auto issue = [&](int k, uint32_t valid) {
        if (lane == 0) vring[k & 3] = valid;
        const int t0 = time_chunk(k) * kChunkT;
        if (tid == 0 && valid != 0u) {
            const int s = k % S;
            pending |= 1u << s;
            uint8_t* st = smem + s * Lay::STAGE;
            mbar_arrive_expect_tx(&full[s], Lay::STAGE);
            tma_load_4d(st, &map_u, &full[s], j0, 0, bd, t0);
            tma_load_3d(st + Lay::U_BYTES, &map_x, &full[s], j0, b, t0);
        }
    };
    if (tid < 32)
        for (int k = 0; k < kAhead && k < nch; ++k)
            issue(k, chunk_valid_bits(mask, time_chunk(k) * kChunkT, L, B, b, lane));
    __syncthreads();

    uint32_t phase_bits = 0;
    const size_t h_tstride = (size_t)B * n_dir * d;
    for (int k = 0; k < nch; ++k) {
        const int s = k % S;
        const int tc = time_chunk(k), t0 = tc * kChunkT;
        const uint32_t valid = vring[k & 3];
        // this lane's row of the chunk whose loads go out at the end of this iteration
        const bool row_next = k + kAhead < nch && chunk_row_ok(mask, time_chunk(k + kAhead) * kChunkT, L, B, b, lane);
        const uint32_t inrange = chunk_inrange_bits(t0, L);
        if (ckpt != nullptr && jok) store_pair(ckpt + ((size_t)tc * B * n_dir + bd) * d + j, c);
        if (valid != 0u) {
            const bool ok = mbar_wait(&full[s], (phase_bits >> s) & 1u, kErrTimeoutLoad);
            if (__syncthreads_or(!ok)) {  // a load never landed: give up (error recorded)
                if (tid == 0) {
                    drain_pending_loads<S>(full, pending, phase_bits);
                    if (kStage) bulk_wait_group<0>();  // stores still reading shared memory
                }
                return;
            }
            phase_bits ^= 1u << s;
            pending &= ~(1u << s);
        }
        const UT* us = reinterpret_cast<const UT*>(smem + s * Lay::STAGE);
        const float* xs = reinterpret_cast<const float*>(smem + s * Lay::STAGE + Lay::U_BYTES);
        float* hp = h + (size_t)t0 * h_tstride + (size_t)bd * d + j;
        const bool staged = kStage && valid == (1u << kChunkT) - 1u;
        if (staged) {
            c = fwd_chunk<UT, CJ, true>(us, xs, valid, inrange, c, p, alpha2, dir, hp, h_tstride, jok, cj);
            fence_proxy_async_shared();  // h over the x tile, visible to the TMA unit
        } else {
            c = fwd_chunk<UT, CJ>(us, xs, valid, inrange, c, p, alpha2, dir, hp, h_tstride, jok, cj);
        }
        __syncthreads();  // every thread is done with stage s
        if (kStage && tid == 0) {
            if (staged) {
                tma_store_3d(&map_h, smem + s * Lay::STAGE + Lay::U_BYTES, j0, bd, t0);
                bulk_commit_group();
            }
            // the next load goes to the stage chunk k-1 used (kAhead = S - 1 here): its
            // store must be done reading it
            if (k + kAhead < nch) {
                if (staged) bulk_wait_group_read<1>();
                else bulk_wait_group_read<0>();
            }
        }
        if (tid < 32 && k + kAhead < nch) issue(k + kAhead, chunk_vote(row_next));
    }
    if (kStage && tid == 0) bulk_wait_group<0>();  // every store has landed
    if (jok) store_pair(c_T + (size_t)bd * d + j, c);
}

// fp64 totals of a thread's dv/db partial sums, acc[q][e] for
// q in {dv_f, dv_r, db_f, db_r} and channel e of the pair: in registers, or
// (SmemPartials) in shared memory, thread-interleaved, so that they hold no
// registers across a long chunk loop.
__device__ __forceinline__ void fold_partials(double (&acc)[4][2], const float2 (&s)[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        acc[q][0] += (double)s[q].x;
        acc[q][1] += (double)s[q].y;
    }
}
struct SmemPartials {
    double* p;  // this thread's first total; total k at p[k * n]
    int n;      // threads of the CTA
};
__device__ __forceinline__ void fold_partials(SmemPartials& acc, const float2 (&s)[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        acc.p[(2 * q) * acc.n] += (double)s[q].x;
        acc.p[(2 * q + 1) * acc.n] += (double)s[q].y;
    }
}

// ---------------------------------------------------------------- backward
// Backward over one chunk staged in shared memory (us, xs, dhs), given the
// state c entering the chunk in forward order and the state gradient g leaving
// it.  With ACC_DX the highway gradient is added onto the dx the other
// direction already wrote (one atomic add per element, after that launch
// completed on the same stream: the same single fp32 addition every run).
// Re-runs the forward over the chunk keeping c, f and r in registers, then
// walks it in reverse: writes dU and dx for the rows that exist, accumulates
// the dv/db partial sums in acc[q] = {dv_f, dv_r, db_f, db_r} (per channel of
// the pair), and updates g.
template <typename UT, typename DUT, bool ACC_DX, int DIR, int CJ = kRecCJ, typename ACC>
__device__ __forceinline__ void bwd_chunk_any(const UT* __restrict__ us, const float* __restrict__ xs,
                                          const float* __restrict__ dhs,
                                          uint32_t valid, uint32_t inrange, float2 c, const GateParams2& p,
                                          float2 alpha, float2& g, ACC& acc, DUT* __restrict__ dUp,
                                          float* __restrict__ dxp, size_t u_tstride, size_t x_tstride, int d,
                                          bool jok, int cj) {
    constexpr uint32_t kFull = (1u << kChunkT) - 1u;
    const bool full = valid == kFull;
    float2 cp[kChunkT], fs[kChunkT], rs[kChunkT];
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = DIR == 0 ? q : kChunkT - 1 - q;
        cp[i] = c;
        fs[i] = f2(0.f);
        rs[i] = f2(0.f);
        if (full || ((valid >> i) & 1u))
            c = sru_cell2(c, load_pair(us + (i * 3 + 0) * CJ + cj), load_pair(us + (i * 3 + 1) * CJ + cj),
                          load_pair(us + (i * 3 + 2) * CJ + cj), p, fs[i], rs[i]);
    }
    // chunk partial sums in fp32 (16 terms), folded into the fp64 totals once per chunk
    float2 s_vf = f2(0.f), s_vr = f2(0.f), s_bf = f2(0.f), s_br = f2(0.f);
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = DIR == 0 ? kChunkT - 1 - q : q;
        if (!full && !((inrange >> i) & 1u)) continue;
        float2 duc = f2(0.f), dzf = f2(0.f), dzr = f2(0.f), dxv = f2(0.f);
        const bool row = full || ((valid >> i) & 1u);
        if (row) {
            const float2 f = fs[i], r = rs[i], cpv = cp[i];
            const float2 uc = load_pair(us + (i * 3 + 0) * CJ + cj);
            const float2 ax = mul2(alpha, load_pair(xs + i * CJ + cj));
            const float2 dhv = load_pair(dhs + i * CJ + cj);
            const float2 cmu = sub2(cpv, uc);
            const float2 cn = fma2(f, cmu, uc);
            const float2 G = fma2(dhv, r, g);  // dLoss/dc[t]
            const float2 omr = sub2(f2(1.f), r), omf = sub2(f2(1.f), f);
            dxv = mul2(mul2(dhv, omr), alpha);
            dzf = mul2(mul2(G, cmu), mul2(f, omf));
            dzr = mul2(mul2(dhv, sub2(cn, ax)), mul2(r, omr));
            duc = mul2(G, omf);
            g = fma2(dzr, p.vr, fma2(dzf, p.vf, mul2(G, f)));  // dLoss/dc[t-1]
            s_vf = fma2(dzf, cpv, s_vf);
            s_vr = fma2(dzr, cpv, s_vr);
            s_bf = add2(s_bf, dzf);
            s_br = add2(s_br, dzr);
        }
        if (jok) {
            store_pair(dUp + (size_t)i * u_tstride, duc);
            store_pair(dUp + (size_t)i * u_tstride + d, dzf);
            store_pair(dUp + (size_t)i * u_tstride + 2 * d, dzr);
            if (ACC_DX) {
                if (row) add_pair(dxp + (size_t)i * x_tstride, dxv);
            } else {
                store_pair(dxp + (size_t)i * x_tstride, dxv);
            }
        }
    }
    const float2 s4[4] = {s_vf, s_vr, s_bf, s_br};
    fold_partials(acc, s4);
}

// Fast path of bwd_chunk for a chunk whose 16 rows all exist and are valid:
// the state chain's operands are copied from shared memory into registers
// before the chain runs, and no row carries a predicate.
// STAGE (DUT == UT): dU and dx are not stored to global memory here but
// written over this thread's own U and x values in the chunk's shared-memory
// stage (same layout; the values were copied to registers first), for the
// caller to send out with two TMA stores.
template <typename UT, typename DUT, bool ACC_DX, int DIR, int CJ, typename ACC, bool STAGE = false>
__device__ __forceinline__ void bwd_chunk_full(const UT* __restrict__ us, const float* __restrict__ xs,
                                               const float* __restrict__ dhs,
                                               float2 c, const GateParams2& p, float2 alpha, float2& g,
                                               ACC& acc, DUT* __restrict__ dUp, float* __restrict__ dxp,
                                               size_t u_tstride, size_t x_tstride, int d, bool jok, int cj) {
    static_assert(!STAGE || sizeof(DUT) == sizeof(UT), "staged dU reuses the U tile");
    using PW = PairWord<UT>;
    typename PW::T wc[kChunkT], wf[kChunkT], wr[kChunkT];
    float2 wx[kChunkT], wdh[kChunkT];
#pragma unroll
    for (int i = 0; i < kChunkT; ++i) {
        wc[i] = PW::load(us + (i * 3 + 0) * CJ + cj);
        wf[i] = PW::load(us + (i * 3 + 1) * CJ + cj);
        wr[i] = PW::load(us + (i * 3 + 2) * CJ + cj);
        wx[i] = load_pair(xs + i * CJ + cj);
        wdh[i] = load_pair(dhs + i * CJ + cj);
    }
    if (STAGE) asm volatile("" ::: "memory");  // every read of the tile precedes the writes over it
    float2 cp[kChunkT], fs[kChunkT], rs[kChunkT];
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = DIR == 0 ? q : kChunkT - 1 - q;
        cp[i] = c;
        c = sru_cell2(c, PW::unpack(wc[i]), PW::unpack(wf[i]), PW::unpack(wr[i]), p, fs[i], rs[i]);
    }
    float2 s_vf = f2(0.f), s_vr = f2(0.f), s_bf = f2(0.f), s_br = f2(0.f);
#pragma unroll
    for (int q = 0; q < kChunkT; ++q) {
        const int i = DIR == 0 ? kChunkT - 1 - q : q;
        const float2 f = fs[i], r = rs[i], cpv = cp[i];
        const float2 uc = PW::unpack(wc[i]);
        const float2 ax = mul2(alpha, wx[i]);
        const float2 dhv = wdh[i];
        const float2 cmu = sub2(cpv, uc);
        const float2 cn = fma2(f, cmu, uc);
        const float2 G = fma2(dhv, r, g);  // dLoss/dc[t]
        const float2 omr = sub2(f2(1.f), r), omf = sub2(f2(1.f), f);
        const float2 dxv = mul2(mul2(dhv, omr), alpha);
        const float2 dzf = mul2(mul2(G, cmu), mul2(f, omf));
        const float2 dzr = mul2(mul2(dhv, sub2(cn, ax)), mul2(r, omr));
        const float2 duc = mul2(G, omf);
        g = fma2(dzr, p.vr, fma2(dzf, p.vf, mul2(G, f)));  // dLoss/dc[t-1]
        s_vf = fma2(dzf, cpv, s_vf);
        s_vr = fma2(dzr, cpv, s_vr);
        s_bf = add2(s_bf, dzf);
        s_br = add2(s_br, dzr);
        if (STAGE) {
            DUT* su = reinterpret_cast<DUT*>(const_cast<UT*>(us));
            store_pair(su + (i * 3 + 0) * CJ + cj, duc);
            store_pair(su + (i * 3 + 1) * CJ + cj, dzf);
            store_pair(su + (i * 3 + 2) * CJ + cj, dzr);
            store_pair(const_cast<float*>(xs) + i * CJ + cj, dxv);
        } else if (jok) {
            store_pair(dUp + (size_t)i * u_tstride, duc);
            store_pair(dUp + (size_t)i * u_tstride + d, dzf);
            store_pair(dUp + (size_t)i * u_tstride + 2 * d, dzr);
            if (ACC_DX)
                add_pair(dxp + (size_t)i * x_tstride, dxv);
            else
                store_pair(dxp + (size_t)i * x_tstride, dxv);
        }
    }
    const float2 s4[4] = {s_vf, s_vr, s_bf, s_br};
    fold_partials(acc, s4);
}

template <typename UT, typename DUT, bool ACC_DX, int DIR, int CJ = kRecCJ, typename ACC>
__device__ __forceinline__ void bwd_chunk(const UT* __restrict__ us, const float* __restrict__ xs,
                                          const float* __restrict__ dhs,
                                          uint32_t valid, uint32_t inrange, float2 c, const GateParams2& p,
                                          float2 alpha, float2& g, ACC& acc, DUT* __restrict__ dUp,
                                          float* __restrict__ dxp, size_t u_tstride, size_t x_tstride, int d,
                                          bool jok, int cj) {
    if (valid == (1u << kChunkT) - 1u)
        bwd_chunk_full<UT, DUT, ACC_DX, DIR, CJ>(us, xs, dhs, c, p, alpha, g, acc, dUp, dxp, u_tstride,
                                                 x_tstride, d, jok, cj);
    else
        bwd_chunk_any<UT, DUT, ACC_DX, DIR, CJ>(us, xs, dhs, valid, inrange, c, p, alpha, g, acc, dUp, dxp,
                                                u_tstride, x_tstride, d, jok, cj);
}

// A chunk with no valid row: zero dU (and dx unless accumulating); g passes through.
template <typename DUT, bool ACC_DX>
__device__ __forceinline__ void bwd_chunk_padded(uint32_t inrange, DUT* __restrict__ dUp, float* __restrict__ dxp,
                                                 size_t u_tstride, size_t x_tstride, int d, bool jok) {
    if (!jok) return;
#pragma unroll
    for (int i = 0; i < kChunkT; ++i) {
        if (!((inrange >> i) & 1u)) continue;
        store_pair(dUp + (size_t)i * u_tstride, f2(0.f));
        store_pair(dUp + (size_t)i * u_tstride + d, f2(0.f));
        store_pair(dUp + (size_t)i * u_tstride + 2 * d, f2(0.f));
        if (!ACC_DX) store_pair(dxp + (size_t)i * x_tstride, f2(0.f));
    }
}

// Per-thread dv/db totals of a channel pair -> partial[row][q][j .. j+1]
__device__ __forceinline__ void store_partials(double* __restrict__ pp, const double (&acc)[4][2], int d) {
#pragma unroll
    for (int q = 0; q < 4; ++q) *reinterpret_cast<double2*>(pp + (size_t)q * d) = make_double2(acc[q][0], acc[q][1]);
}
__device__ __forceinline__ void store_partials(double* __restrict__ pp, const SmemPartials& acc, int d) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<double2*>(pp + (size_t)q * d) = make_double2(acc.p[(2 * q) * acc.n], acc.p[(2 * q + 1) * acc.n]);
}

template <typename UT, bool ACC_DX, int CJ = kRecCJ, int S = kBwdStages>
struct BwdLayout {
    static constexpr int U_BYTES = kChunkT * 3 * CJ * (int)sizeof(UT);
    static constexpr int V_BYTES = kChunkT * CJ * 4;  // one fp32 (T, CJ) tile
    static constexpr int STAGE = U_BYTES + 2 * V_BYTES;  // U, x, dh
    static constexpr int ACC_OFF = S * STAGE;  // SmemPartials: 8 doubles per thread
    static constexpr int BAR_OFF = ACC_OFF + (CJ / 2) * 8 * 8;
    static constexpr int SMEM = BAR_OFF + 64 + 128;
};

// Backward of direction DIR.  Grid (ceil(d/CJ), B), CJ/2 threads (CJ/64 warps) per CTA.
// ACC_DX: dx += this direction's highway gradient (dx already holds the other
// direction's, written by an earlier launch on the same stream), else dx = it.
// Adding with 8-byte atomics instead of staging dx keeps a stage at U + x + dh,
// so as many CTAs fit on an SM as in the first direction's launch.
//   map_dh: 3-D (d, B*n_dir, L) fp32.
// DIR is a template parameter so the per-chunk register arrays are indexed
// with compile-time constants.
template <typename UT, typename DUT, bool ACC_DX, int DIR, int CJ, int S>
__global__ void __launch_bounds__(CJ / 2) sru_bwd_seq_kernel(
    const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_x,
    const __grid_constant__ CUtensorMap map_dh, const __grid_constant__ CUtensorMap map_du,
    const __grid_constant__ CUtensorMap map_dxo, const float* __restrict__ v, const float* __restrict__ bias,
    const uint8_t* __restrict__ mask, const float* __restrict__ ckpt, const float* __restrict__ dc_T, DUT* __restrict__ dU,
    float* __restrict__ dx, double* __restrict__ partial, float* __restrict__ dc0, const int* __restrict__ order, int L,
    int B, int d, int n_dir, float alpha) {
    using Lay = BwdLayout<UT, ACC_DX, CJ, S>;
    // Full chunks leave through TMA stores of the stage they came in on (dU over
    // U, dx over x).  With S >= 3 a stage is refilled one iteration after its
    // store was issued, so loads run S - 1 chunks ahead; with S = 2 loads run 2
    // ahead and the stage just stored is refilled as soon as its store has read
    // it (a wait of a few hundred cycles).
    constexpr bool kStage = sizeof(UT) == sizeof(DUT) && S >= 2;
    constexpr int kAhead = S >= 3 ? S - 1 : S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);

    const int tid = threadIdx.x, lane = tid & 31, cj = 2 * tid;
    const int j0 = blockIdx.x * CJ, j = j0 + cj;
    constexpr int dir = DIR;
    // with `order`, the batch rows longest first (its entries are (b, dir) streams, n_dir per row)
    const int b = order != nullptr ? order[blockIdx.y * n_dir] / n_dir : (int)blockIdx.y;
    const int bd = b * n_dir + dir;
    const bool jok = j < d;
    const int nch = (L + kChunkT - 1) / kChunkT;

    GateParams2 p = make_gate_params2(f2(0.f), f2(0.f), f2(0.f), f2(0.f));
    float2 g = f2(0.f);
    if (jok) {
        p = make_gate_params2(load_pair(v + (dir * 2 + 0) * d + j), load_pair(v + (dir * 2 + 1) * d + j),
                              load_pair(bias + (dir * 2 + 0) * d + j), load_pair(bias + (dir * 2 + 1) * d + j));
        if (dc_T != nullptr) g = load_pair(dc_T + (size_t)bd * d + j);
    }
    const float2 alpha2 = f2(alpha);
    if (tid == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
        tma_prefetch_desc(&map_u);
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_dh);
        if (kStage) {
            tma_prefetch_desc(&map_du);
            tma_prefetch_desc(&map_dxo);
        }
    }
    __syncthreads();

    // backward processing chunk k covers time chunk: dir 0 walks time chunks downwards
    auto time_chunk = [&](int k) { return dir == 0 ? nch - 1 - k : k; };
    // the row-validity words of processing chunks k .. k + kAhead, slot k & 3: each is
    // voted on when its chunk's loads are issued, from mask bytes fetched one chunk
    // earlier, so no mask read sits on the chain
    uint32_t* vring = reinterpret_cast<uint32_t*>(full + S);
    uint32_t pending = 0;  // thread 0: stages with a load in flight
    auto issue = [&](int k, uint32_t valid) {
        if (lane == 0) vring[k & 3] = valid;
        const int t0 = time_chunk(k) * kChunkT;
        if (tid == 0 && valid != 0u) {
            const int s = k % S;
            pending |= 1u << s;
            uint8_t* st = smem + s * Lay::STAGE;
            mbar_arrive_expect_tx(&full[s], Lay::STAGE);
            tma_load_4d(st, &map_u, &full[s], j0, 0, bd, t0);
            tma_load_3d(st + Lay::U_BYTES, &map_x, &full[s], j0, b, t0);
            tma_load_3d(st + Lay::U_BYTES + Lay::V_BYTES, &map_dh, &full[s], j0, bd, t0);
        }
    };
    if (tid < 32)
        for (int k = 0; k < kAhead && k < nch; ++k)
            issue(k, chunk_valid_bits(mask, time_chunk(k) * kChunkT, L, B, b, lane));
    __syncthreads();

    SmemPartials acc{reinterpret_cast<double*>(smem + Lay::ACC_OFF) + tid, CJ / 2};
#pragma unroll
    for (int q = 0; q < 8; ++q) acc.p[q * acc.n] = 0.0;  // read and written by this thread only
    uint32_t phase_bits = 0;
    const size_t u_tstride = (size_t)B * n_dir * 3 * d;
    const size_t x_tstride = (size_t)B * d;
    // Checkpoint (state entering the chunk in time order) of backward chunk k.
    // Loaded two chunks ahead of use so its global-memory latency is not on
    // the chain.
    auto ckpt_of = [&](int k) {
        return (jok && k < nch) ? load_pair(ckpt + ((size_t)time_chunk(k) * B * n_dir + bd) * d + j) : f2(0.f);
    };
    // Waits for stage s's load; on expiry every thread leaves (after lane 0
    // drained the loads in flight).
    auto wait_stage = [&](int s) {
        const bool ok = mbar_wait(&full[s], (phase_bits >> s) & 1u, kErrTimeoutLoad);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                drain_pending_loads<S>(full, pending, phase_bits);
                if (kStage) bulk_wait_group<0>();  // stores still reading shared memory
            }
            return false;
        }
        return true;
    };
    float2 ck0 = ckpt_of(0), ck1 = ckpt_of(1);
    for (int k = 0; k < nch; ++k) {
        const int s = k % S;
        const int tc = time_chunk(k), t0 = tc * kChunkT;
        const uint32_t valid = vring[k & 3];
        // this lane's row of the chunk whose loads go out at the end of this iteration
        const bool row_next = k + kAhead < nch && chunk_row_ok(mask, time_chunk(k + kAhead) * kChunkT, L, B, b, lane);
        const uint32_t inrange = chunk_inrange_bits(t0, L);
        const float2 ck2 = ckpt_of(k + 2);
        DUT* dUp = dU + (size_t)t0 * u_tstride + (size_t)bd * 3 * d + j;
        float* dxp = dx + (size_t)t0 * x_tstride + (size_t)b * d + j;
        bool staged = false;
        if (valid == 0u) {
            bwd_chunk_padded<DUT, ACC_DX>(inrange, dUp, dxp, u_tstride, x_tstride, d, jok);
        } else {
            if (!wait_stage(s)) return;
            phase_bits ^= 1u << s;
            pending &= ~(1u << s);
            const UT* us = reinterpret_cast<const UT*>(smem + s * Lay::STAGE);
            const float* xs = reinterpret_cast<const float*>(smem + s * Lay::STAGE + Lay::U_BYTES);
            const float* dhs = xs + kChunkT * CJ;
            if constexpr (kStage) {
                if (valid == (1u << kChunkT) - 1u) {
                    bwd_chunk_full<UT, DUT, ACC_DX, DIR, CJ, SmemPartials, true>(us, xs, dhs, ck0, p, alpha2, g, acc,
                                                                                 dUp, dxp, u_tstride, x_tstride, d,
                                                                                 jok, cj);
                    fence_proxy_async_shared();  // the tile's new contents, visible to the TMA unit
                    staged = true;
                }
            }
            if (!staged)
                bwd_chunk<UT, DUT, ACC_DX, DIR, CJ>(us, xs, dhs, valid, inrange, ck0, p, alpha2, g, acc, dUp, dxp,
                                                    u_tstride, x_tstride, d, jok, cj);
        }
        __syncthreads();
        if (kStage && tid == 0) {
            if (staged) {
                const uint8_t* st = smem + s * Lay::STAGE;
                tma_store_4d(&map_du, st, j0, 0, bd, t0);
                if (ACC_DX)
                    tma_reduce_add_3d(&map_dxo, st + Lay::U_BYTES, j0, b, t0);
                else
                    tma_store_3d(&map_dxo, st + Lay::U_BYTES, j0, b, t0);
                bulk_commit_group();
            }
            if (k + kAhead < nch) {
                if (kAhead == S) {
                    // the next load goes to this chunk's stage: its store must be done reading it
                    if (staged) bulk_wait_group_read<0>();
                } else if (staged) {
                    // the next load goes to the stage chunk k-1 used: its store must be done reading it
                    bulk_wait_group_read<1>();
                } else {
                    bulk_wait_group_read<0>();
                }
            }
        }
        if (tid < 32 && k + kAhead < nch) issue(k + kAhead, chunk_vote(row_next));
        ck0 = ck1;
        ck1 = ck2;
    }
    if (kStage && tid == 0) bulk_wait_group<0>();  // every store has landed
    if (jok) {
        store_pair(dc0 + (size_t)bd * d + j, g);
        store_partials(partial + (size_t)bd * 4 * d + j, acc, d);
    }
}

// dv, db = sum over rows of the per-row partial sums.  partial: (rows,
// n_dir, 4, d) doubles, [dv_f, dv_r, db_f, db_r].  A block owns
// kRedCols consecutive output columns; its kRedSlices row slices each sum
// rows slice, slice + kRedSlices, ... in increasing order, and the slices are
// then added in increasing order: a fixed order, so the result is the same
// on every run.
constexpr int kRedCols = 32, kRedSlices = 8;
__global__ void __launch_bounds__(kRedCols * kRedSlices) sru_reduce_dvdb_kernel(
    const double* __restrict__ partial, int rows, int d, int n_dir, float* __restrict__ dv, float* __restrict__ db) {
    __shared__ double part[kRedSlices][kRedCols];
    const int col = threadIdx.x % kRedCols, slice = threadIdx.x / kRedCols;
    const int idx = blockIdx.x * kRedCols + col;
    const int ncols = n_dir * 4 * d;
    double s = 0.0;
    if (idx < ncols)
        for (int rr = slice; rr < rows; rr += kRedSlices) s += partial[(size_t)rr * ncols + idx];
    part[slice][col] = s;
    __syncthreads();
    if (slice != 0 || idx >= ncols) return;
    double t = 0.0;
#pragma unroll
    for (int k = 0; k < kRedSlices; ++k) t += part[k][col];
    const int dir = idx / (4 * d), q = (idx / d) % 4, j = idx % d;
    if (q < 2)
        dv[(dir * 2 + q) * d + j] = (float)t;
    else
        db[(dir * 2 + q - 2) * d + j] = (float)t;
}

// Launch order of a padded layer's (batch row, direction) streams, longest
// first.  A row's work is its number of kChunkT-step chunks holding a valid
// (unpadded) step: padded chunks cost only their zero outputs.  With every
// CTA walking a whole sequence, taking the long rows first lets the short ones
// fill the SMs behind them (longest-processing-time-first), instead of each
// wave of resident CTAs lasting as long as its longest row.  One block; rows
// of equal work keep their index order, so the order is deterministic.
//   order[r * n_dir + dir] = b * n_dir + dir for the row b of rank r.
constexpr int kOrderThreads = 1024;
constexpr int kOrderMaxB = 2048;
__global__ void __launch_bounds__(kOrderThreads) sru_length_order_kernel(const uint8_t* __restrict__ mask, int L,
                                                                         int B, int n_dir, int* __restrict__ order) {
    __shared__ int work[kOrderMaxB];
    const int nch = (L + kChunkT - 1) / kChunkT;
    for (int b = threadIdx.x; b < B; b += blockDim.x) work[b] = 0;
    __syncthreads();
    for (long long idx = threadIdx.x; idx < (long long)B * nch; idx += blockDim.x) {
        const int b = (int)(idx % B), c = (int)(idx / B);  // consecutive threads: consecutive rows, coalesced
        const int t1 = min(L, (c + 1) * kChunkT);
        bool any = false;
        for (int t = c * kChunkT; t < t1; ++t) any |= mask[(size_t)t * B + b] == 0;
        if (any) atomicAdd(&work[b], 1);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const int wb = work[b];
        int rank = 0;
        for (int o = 0; o < B; ++o) {
            const int wo = work[o];
            rank += (wo > wb) || (wo == wb && o < b);
        }
        for (int dir = 0; dir < n_dir; ++dir) order[rank * n_dir + dir] = b * n_dir + dir;
    }
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
