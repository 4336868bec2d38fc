// sru_scan.cuh -- the linear case v = 0 of the SRU recurrence as a chunked
// associative scan over t.
//
// With v_f = v_r = 0 the gates of Eqs. (2)-(3) no longer read c[t-1]
// ("When Attention Meets Fast Recurrence", background section on SRU), so
// Eq. (4) is a first-order linear recurrence c[t] = f[t] c[t-1] + (1-f[t]) u[t]
// and a chunk of steps acts on the state as an affine map c -> A c + Bc with
// A = prod f.  Linear recurrent layers can be trained in parallel over time
// ("Parallelizing Legendre Memory Unit Training", abstract); here time is cut
// into chunks of kScanT steps so that B*d channels x L/kScanT chunks of work
// exist even when B*d alone cannot fill the GPU.
//
// One CTA = one (chunk, 64-channel tile).  It stages its chunk in shared
// memory with TMA, reduces it to (A, Bc), publishes that aggregate, and finds
// the state entering the chunk by a decoupled look-back over its predecessors
// (each publishes its aggregate, then its inclusive prefix).  Work items are
// handed out by an atomic ticket in chunk-major order, so every predecessor a
// CTA waits on was started earlier by a resident CTA: the waits always end.
// They are bounded anyway; an expired wait publishes an abort flag that
// releases every successor, records kErrTimeoutScan and returns.
// The chunk is then walked again from shared memory with the carried-in state
// (forward: h, checkpoints; backward: dU, dx, dv/db partials).
// The backward uses the same scheme on the state gradient g = dLoss/dc, whose
// recurrence is affine in g for ANY v (the peepholes only make its
// coefficients depend on the forward state, which each chunk recomputes from
// the forward's checkpoints): g[t-1] = a[t] g[t] + b[t].  So the backward scan
// serves every layer whose sequential grid would underfill the GPU, not only
// v = 0; the forward scan needs v = 0.
#pragma once

#include "sru_recurrence.cuh"

namespace sru {

constexpr int kScanSub = 8;                 // 16-step sub-chunks per scan chunk
constexpr int kScanT = kScanSub * kChunkT;  // steps per scan chunk

enum ScanFlag : unsigned { kFlagNone = 0, kFlagAgg = 1, kFlagPrefix = 2, kFlagAbort = 3 };

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ float2 ld_relaxed_gpu2(const float* p) {
    float2 v;
    asm volatile("ld.relaxed.gpu.global.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p) : "memory");
    return v;
}

struct ScanState {
    unsigned* flags;  // n_items flags, then the ticket counter
    float* agg_a;     // n_items * CJ (one value per channel)
    float* agg_b;
    float* prefix;
    int withhold;     // item that publishes no carry (fault injection for tests); -1 = none
};

// Whole CTA: publish this item's value(s) (already stored by every thread) under flag f.
__device__ __forceinline__ void scan_publish(unsigned* flag, unsigned f) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        st_release_gpu(flag, f);
    }
}

// Whole CTA: wait (bounded) until flag != 0; returns its value (kFlagAbort on timeout).
__device__ __forceinline__ unsigned scan_wait_flag(const unsigned* flag, unsigned* s_flag) {
    if (threadIdx.x == 0) {
        unsigned f = ld_acquire_gpu(flag);
        if (f == kFlagNone) {
            const uint64_t t0 = globaltimer_ns();
            while ((f = ld_acquire_gpu(flag)) == kFlagNone) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    record_error(kErrTimeoutScan);
                    f = kFlagAbort;
                    break;
                }
                __nanosleep(64);
            }
        }
        *s_flag = f;
    }
    __syncthreads();
    const unsigned f = *s_flag;
    __syncthreads();
    return f;
}

// Decoupled look-back: the composition of the affine maps of items
// k-1, k-2, ... (same tile) applied to the first available inclusive prefix,
// for this thread's channel pair (offset cj).  Returns false on abort.
__device__ __forceinline__ bool scan_lookback(const ScanState& ss, int k, int tile, int n_tiles, int cj,
                                              unsigned* s_flag, float2& carry) {
    float2 a_acc = f2(1.f), b_acc = f2(0.f);
    for (int p = k - 1; p >= 0; --p) {
        const size_t item = (size_t)p * n_tiles + tile;
        const unsigned f = scan_wait_flag(&ss.flags[item], s_flag);
        if (f == kFlagAbort) return false;
        if (f == kFlagPrefix) {
            carry = fma2(a_acc, ld_relaxed_gpu2(&ss.prefix[item * kRecCJ + cj]), b_acc);
            return true;
        }
        const float2 a = ld_relaxed_gpu2(&ss.agg_a[item * kRecCJ + cj]);
        const float2 bb = ld_relaxed_gpu2(&ss.agg_b[item * kRecCJ + cj]);
        b_acc = fma2(a_acc, bb, b_acc);
        a_acc = mul2(a_acc, a);
    }
    carry = b_acc;  // unreachable in practice: item 0 always publishes a prefix
    return true;
}

// Zero the flags and the ticket counter before a scan launch.
__global__ void sru_scan_reset_kernel(unsigned* __restrict__ flags, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) flags[i] = 0u;
}

// A scan CTA has one warp per 16-step sub-chunk of its item: warp q stages,
// reduces and re-walks sub-chunk q, so the item's 128 dependent steps run as
// eight chains of 16 in parallel.  The sub-chunks' affine maps meet in shared
// memory (one float4 (A.x, A.y, B.x, B.y) per lane and sub-chunk) and are
// composed there, in the direction's time order, into the item's map and into
// the state entering each sub-chunk.
constexpr int kScanThreads = kScanSub * 32;

// (A, B) of the maps applied one after another: first (a0, b0), then (a1, b1).
__device__ __forceinline__ void compose_after(float2& a0, float2& b0, float2 a1, float2 b1) {
    b0 = fma2(a1, b0, b1);
    a0 = mul2(a1, a0);
}

template <typename UT>
struct FwdScanLayout {
    static constexpr int STAGE = FwdLayout<UT>::STAGE;
    static constexpr int MAP_OFF = kScanSub * STAGE;
    static constexpr int BAR_OFF = MAP_OFF + kScanSub * 32 * 16;
    static constexpr int SMEM = BAR_OFF + kScanSub * 8 + 64 + 128;
};

// Forward, v = 0.  1-D grid of n_items = ceil(L/kScanT) * ceil(d/CJ) * B * n_dir
// CTAs of kScanThreads threads.
template <typename UT>
__global__ void __launch_bounds__(kScanThreads) sru_fwd_scan_kernel(
    const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_x,
    const float* __restrict__ bias, const float* __restrict__ c0, const uint8_t* __restrict__ mask,
    float* __restrict__ h, float* __restrict__ c_T, float* __restrict__ ckpt, ScanState ss, int L, int B, int d,
    int n_dir, float alpha) {
    using Lay = FwdScanLayout<UT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float4* s_map = reinterpret_cast<float4*>(smem + Lay::MAP_OFF);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);    // one per sub-chunk
    unsigned* s_misc = reinterpret_cast<unsigned*>(bar + kScanSub);       // [0] ticket, [1] flag

    const int tid = threadIdx.x, q = tid >> 5, lane = tid & 31, cj = 2 * lane;
    const int n_jt = (d + kRecCJ - 1) / kRecCJ;
    const int n_tiles = n_jt * B * n_dir;
    const int n_items = gridDim.x;
    if (tid == 0) {
        s_misc[0] = atomicAdd(&ss.flags[n_items], 1u);
        for (int i = 0; i < kScanSub; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int w = (int)s_misc[0];
    const int k = w / n_tiles, tile = w % n_tiles;
    const int jt = tile % n_jt, bd = tile / n_jt;
    const int b = bd / n_dir, dir = bd % n_dir;
    const int nchs = (L + kScanT - 1) / kScanT;
    const int tc = dir == 0 ? k : nchs - 1 - k;
    const int t0 = tc * kScanT;
    const int j0 = jt * kRecCJ, j = j0 + cj;
    const bool jok = j < d;
    const int nch16 = (L + kChunkT - 1) / kChunkT;

    GateParams2 p = make_gate_params2(f2(0.f), f2(0.f), f2(0.f), f2(0.f));
    if (jok)
        p = make_gate_params2(f2(0.f), f2(0.f), load_pair(bias + (dir * 2 + 0) * d + j),
                              load_pair(bias + (dir * 2 + 1) * d + j));
    // this warp's sub-chunk: rows ts .. ts + 15
    const int ts = t0 + q * kChunkT;
    const uint32_t valid = ts < L ? chunk_valid_bits(mask, ts, L, B, b, lane) : 0u;
    const uint32_t inrange = ts < L ? chunk_inrange_bits(ts, L) : 0u;
    uint8_t* st = smem + q * Lay::STAGE;
    if (lane == 0 && valid != 0u) {
        mbar_arrive_expect_tx(&bar[q], (uint32_t)Lay::STAGE);
        tma_load_4d(st, &map_u, &bar[q], j0, 0, bd, ts);
        tma_load_3d(st + FwdLayout<UT>::U_BYTES, &map_x, &bar[q], j0, b, ts);
    }
    const bool ok = valid == 0u || mbar_wait(&bar[q], 0, kErrTimeoutLoad);
    if (__syncthreads_or(!ok)) {
        if (lane == 0 && valid != 0u) mbar_wait(&bar[q], 0, kErrTimeoutLoad);
        scan_publish(&ss.flags[w], kFlagAbort);
        return;
    }

    // 1. this sub-chunk as an affine map of its entering state, then the item's
    const UT* us = reinterpret_cast<const UT*>(st);
    float2 A = f2(1.f), Bc = f2(0.f);
#pragma unroll
    for (int r = 0; r < kChunkT; ++r) {
        const int i = dir == 0 ? r : kChunkT - 1 - r;
        if ((valid >> i) & 1u) {
            const float2 uc = load_pair(us + (i * 3 + 0) * kRecCJ + cj);
            const float2 f = sigmoid2_nl2(fma2(load_pair(us + (i * 3 + 1) * kRecCJ + cj), f2(kNegLog2e), p.nbf));
            A = mul2(A, f);
            Bc = fma2(f, sub2(Bc, uc), uc);
        }
    }
    s_map[q * 32 + lane] = make_float4(A.x, A.y, Bc.x, Bc.y);
    __syncthreads();
    // item map and the map of the sub-chunks before this one, in time order
    float2 Ai = f2(1.f), Bi = f2(0.f), Ab = f2(1.f), Bb = f2(0.f);
#pragma unroll
    for (int qq = 0; qq < kScanSub; ++qq) {
        const int qs = dir == 0 ? qq : kScanSub - 1 - qq;
        if (qs == q) {
            Ab = Ai;
            Bb = Bi;
        }
        const float4 m = s_map[qs * 32 + lane];
        compose_after(Ai, Bi, make_float2(m.x, m.y), make_float2(m.z, m.w));
    }
    // 2. state entering the item
    float2 c_in = f2(0.f);
    const size_t me = (size_t)w * kRecCJ + cj;
    if (k == 0) {
        c_in = (jok && c0 != nullptr) ? load_pair(c0 + (size_t)bd * d + j) : f2(0.f);
    } else {
        if (q == 0) {
            store_pair(ss.agg_a + me, Ai);
            store_pair(ss.agg_b + me, Bi);
        }
        scan_publish(&ss.flags[w], kFlagAgg);
        if (!scan_lookback(ss, k, tile, n_tiles, cj, s_misc + 1, c_in)) {
            scan_publish(&ss.flags[w], kFlagAbort);
            return;
        }
    }
    if (w == ss.withhold) return;  // successors' waits expire (test hook)
    if (q == 0) store_pair(ss.prefix + me, fma2(Ai, c_in, Bi));
    scan_publish(&ss.flags[w], kFlagPrefix);

    // 3. walk this sub-chunk again from its entering state: h and its checkpoint
    if (ts >= L) return;
    float2 c = fma2(Ab, c_in, Bb);
    const int c16 = tc * kScanSub + q;
    if (ckpt != nullptr && jok && c16 < nch16) store_pair(ckpt + ((size_t)c16 * B * n_dir + bd) * d + j, c);
    const size_t h_tstride = (size_t)B * n_dir * d;
    const float* xs = reinterpret_cast<const float*>(st + FwdLayout<UT>::U_BYTES);
    float* hp = h + (size_t)ts * h_tstride + (size_t)bd * d + j;
    c = fwd_chunk<UT, kRecCJ>(us, xs, valid, inrange, c, p, f2(alpha), dir, hp, h_tstride, jok, cj);
    // the last sub-chunk in walk order leaves c_T
    const bool last = dir == 0 ? (ts + kChunkT >= L || q == kScanSub - 1) : q == 0;
    if (k == nchs - 1 && last && jok) store_pair(c_T + (size_t)bd * d + j, c);
}

template <typename UT, bool ACC_DX>
struct BwdScanLayout {
    static constexpr int STAGE = BwdLayout<UT, ACC_DX>::STAGE;
    static constexpr int ACC_OFF = kScanSub * STAGE;                  // SmemPartials: 8 doubles per thread
    static constexpr int MAP_OFF = ACC_OFF + kScanThreads * 8 * 8;
    static constexpr int BAR_OFF = MAP_OFF + kScanSub * 32 * 16;
    static constexpr int SMEM = BAR_OFF + kScanSub * 8 + 64 + 128;
};

// Backward of direction DIR.  1-D grid of n_items = ceil(L/kScanT) * ceil(d/CJ) * B
// CTAs of kScanThreads threads (warp q: sub-chunk q of the item).
// partial: (nchs * B, n_dir, 4, d) doubles.
template <typename UT, typename DUT, bool ACC_DX, int DIR, bool VZERO>
__global__ void __launch_bounds__(kScanThreads) sru_bwd_scan_kernel(
    const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_x,
    const __grid_constant__ CUtensorMap map_dh,
    const float* __restrict__ v, const float* __restrict__ bias, const uint8_t* __restrict__ mask,
    const float* __restrict__ ckpt, const float* __restrict__ dc_T, DUT* __restrict__ dU, float* __restrict__ dx,
    double* __restrict__ partial, float* __restrict__ dc0, ScanState ss, int L, int B, int d, int n_dir,
    float alpha) {
    using Lay = BwdScanLayout<UT, ACC_DX>;
    using SL = BwdLayout<UT, ACC_DX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float4* s_map = reinterpret_cast<float4*>(smem + Lay::MAP_OFF);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
    unsigned* s_misc = reinterpret_cast<unsigned*>(bar + kScanSub);

    const int tid = threadIdx.x, q = tid >> 5, lane = tid & 31, cj = 2 * lane;
    const int n_jt = (d + kRecCJ - 1) / kRecCJ;
    const int n_tiles = n_jt * B;
    const int n_items = gridDim.x;
    if (tid == 0) {
        s_misc[0] = atomicAdd(&ss.flags[n_items], 1u);
        for (int i = 0; i < kScanSub; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int w = (int)s_misc[0];
    const int k = w / n_tiles, tile = w % n_tiles;
    const int jt = tile % n_jt, b = tile / n_jt;
    const int bd = b * n_dir + DIR;
    const int nchs = (L + kScanT - 1) / kScanT;
    const int tc = DIR == 0 ? nchs - 1 - k : k;  // backward walks direction 0 from the end
    const int t0 = tc * kScanT;
    const int j0 = jt * kRecCJ, j = j0 + cj;
    const bool jok = j < d;

    GateParams2 p = make_gate_params2(f2(0.f), f2(0.f), f2(0.f), f2(0.f));
    if (jok)
        p = make_gate_params2(load_pair(v + (DIR * 2 + 0) * d + j), load_pair(v + (DIR * 2 + 1) * d + j),
                              load_pair(bias + (DIR * 2 + 0) * d + j), load_pair(bias + (DIR * 2 + 1) * d + j));
    const float2 alpha2 = f2(alpha);
    const int nch16 = (L + kChunkT - 1) / kChunkT;
    // this warp's sub-chunk: rows ts .. ts + 15
    const int ts = t0 + q * kChunkT;
    const uint32_t valid = ts < L ? chunk_valid_bits(mask, ts, L, B, b, lane) : 0u;
    const uint32_t inrange = ts < L ? chunk_inrange_bits(ts, L) : 0u;
    uint8_t* st = smem + q * SL::STAGE;
    if (lane == 0 && valid != 0u) {
        mbar_arrive_expect_tx(&bar[q], (uint32_t)SL::STAGE);
        tma_load_4d(st, &map_u, &bar[q], j0, 0, bd, ts);
        tma_load_3d(st + SL::U_BYTES, &map_x, &bar[q], j0, b, ts);
        tma_load_3d(st + SL::U_BYTES + SL::V_BYTES, &map_dh, &bar[q], j0, bd, ts);
    }
    // the sub-chunk's forward checkpoint, fetched while the tiles load
    const int c16 = tc * kScanSub + q;
    const float2 ck = (jok && c16 < nch16) ? load_pair(ckpt + ((size_t)c16 * B * n_dir + bd) * d + j) : f2(0.f);
    const bool ok = valid == 0u || mbar_wait(&bar[q], 0, kErrTimeoutLoad);
    if (__syncthreads_or(!ok)) {
        if (lane == 0 && valid != 0u) mbar_wait(&bar[q], 0, kErrTimeoutLoad);
        scan_publish(&ss.flags[w], kFlagAbort);
        return;
    }
    const UT* us = reinterpret_cast<const UT*>(st);
    const float* xs = reinterpret_cast<const float*>(st + SL::U_BYTES);
    const float* dhs = xs + kChunkT * kRecCJ;

    // 1. this sub-chunk as an affine map of the state gradient, g_out = A g_in + Bg.
    //    Each valid row maps g to a g + b with (see bwd_chunk)
    //      a = f + (c' - u) f(1-f) v_f,  b = a dh r + dh (c - alpha x) r(1-r) v_r,
    //    which needs the row's forward state: the sub-chunk is re-run from its
    //    checkpoint (bit-identical to the forward), then walked back.
    float2 A = f2(1.f), Bg = f2(0.f);
    if (VZERO) {
        // v = 0: the gates do not read c, so a = f and b = f dh r need no state
#pragma unroll
        for (int r = 0; r < kChunkT; ++r) {
            const int i = DIR == 0 ? kChunkT - 1 - r : r;
            if ((valid >> i) & 1u) {
                const float2 f = sigmoid2_nl2(fma2(load_pair(us + (i * 3 + 1) * kRecCJ + cj), f2(kNegLog2e), p.nbf));
                const float2 rr =
                    sigmoid2_nl2(fma2(load_pair(us + (i * 3 + 2) * kRecCJ + cj), f2(kNegLog2e), p.nbr));
                A = mul2(A, f);
                Bg = mul2(f, fma2(load_pair(dhs + i * kRecCJ + cj), rr, Bg));
            }
        }
    } else if (valid != 0u) {
        float2 c = ck;
        float2 cp[kChunkT], fs[kChunkT], rs[kChunkT];
#pragma unroll
        for (int r = 0; r < kChunkT; ++r) {
            const int i = DIR == 0 ? r : kChunkT - 1 - r;
            cp[i] = c;
            fs[i] = f2(0.f);
            rs[i] = f2(0.f);
            if ((valid >> i) & 1u)
                c = sru_cell2(c, load_pair(us + (i * 3 + 0) * kRecCJ + cj), load_pair(us + (i * 3 + 1) * kRecCJ + cj),
                              load_pair(us + (i * 3 + 2) * kRecCJ + cj), p, fs[i], rs[i]);
        }
#pragma unroll
        for (int r = 0; r < kChunkT; ++r) {
            const int i = DIR == 0 ? kChunkT - 1 - r : r;
            if (!((valid >> i) & 1u)) continue;
            const float2 f = fs[i], rr = rs[i];
            const float2 uc = load_pair(us + (i * 3 + 0) * kRecCJ + cj);
            const float2 ax = mul2(alpha2, load_pair(xs + i * kRecCJ + cj));
            const float2 dhv = load_pair(dhs + i * kRecCJ + cj);
            const float2 cmu = sub2(cp[i], uc);
            const float2 cn = fma2(f, cmu, uc);
            const float2 dzr = mul2(mul2(dhv, sub2(cn, ax)), mul2(rr, sub2(f2(1.f), rr)));
            const float2 a = fma2(mul2(cmu, mul2(f, sub2(f2(1.f), f))), p.vf, f);
            const float2 bb = fma2(dzr, p.vr, mul2(a, mul2(dhv, rr)));
            A = mul2(a, A);
            Bg = fma2(a, Bg, bb);
        }
    }
    s_map[q * 32 + lane] = make_float4(A.x, A.y, Bg.x, Bg.y);
    __syncthreads();
    // item map and the map of the sub-chunks walked before this one (backward walk order)
    float2 Ai = f2(1.f), Bi = f2(0.f), Ab = f2(1.f), Bb = f2(0.f);
#pragma unroll
    for (int qq = 0; qq < kScanSub; ++qq) {
        const int qs = DIR == 0 ? kScanSub - 1 - qq : qq;
        if (qs == q) {
            Ab = Ai;
            Bb = Bi;
        }
        const float4 m = s_map[qs * 32 + lane];
        compose_after(Ai, Bi, make_float2(m.x, m.y), make_float2(m.z, m.w));
    }
    // 2. state gradient entering the item (from later times)
    float2 g_in = f2(0.f);
    const size_t me = (size_t)w * kRecCJ + cj;
    if (k == 0) {
        g_in = (jok && dc_T != nullptr) ? load_pair(dc_T + (size_t)bd * d + j) : f2(0.f);
    } else {
        if (q == 0) {
            store_pair(ss.agg_a + me, Ai);
            store_pair(ss.agg_b + me, Bi);
        }
        scan_publish(&ss.flags[w], kFlagAgg);
        if (!scan_lookback(ss, k, tile, n_tiles, cj, s_misc + 1, g_in)) {
            scan_publish(&ss.flags[w], kFlagAbort);
            return;
        }
    }
    if (w == ss.withhold) return;  // successors' waits expire (test hook)
    if (q == 0) store_pair(ss.prefix + me, fma2(Ai, g_in, Bi));
    scan_publish(&ss.flags[w], kFlagPrefix);

    // 3. gradients of this sub-chunk's rows from the state gradient entering it
    float2 g = fma2(Ab, g_in, Bb);
    SmemPartials acc{reinterpret_cast<double*>(smem + Lay::ACC_OFF) + tid, kScanThreads};
#pragma unroll
    for (int i = 0; i < 8; ++i) acc.p[i * acc.n] = 0.0;  // read and written by this thread only
    if (ts < L) {
        const size_t u_tstride = (size_t)B * n_dir * 3 * d;
        const size_t x_tstride = (size_t)B * d;
        DUT* dUp = dU + (size_t)ts * u_tstride + (size_t)bd * 3 * d + j;
        float* dxp = dx + (size_t)ts * x_tstride + (size_t)b * d + j;
        if (valid == 0u)
            bwd_chunk_padded<DUT, ACC_DX>(inrange, dUp, dxp, u_tstride, x_tstride, d, jok);
        else
            bwd_chunk<UT, DUT, ACC_DX, DIR, kRecCJ>(us, xs, dhs, valid, inrange, ck, p, alpha2, g, acc, dUp, dxp,
                                                    u_tstride, x_tstride, d, jok, cj);
    }
    // the last sub-chunk in walk order leaves dc0
    const bool last = DIR == 0 ? q == 0 : (ts + kChunkT >= L || q == kScanSub - 1);
    if (k == nchs - 1 && last && ts < L && jok) store_pair(dc0 + (size_t)bd * d + j, g);
    // the item's dv/db partial sums: the warps' totals in sub-chunk order
    __syncthreads();
    if (q == 0 && jok) {
        const double* base = reinterpret_cast<const double*>(smem + Lay::ACC_OFF);
        double* pp = partial + (((size_t)tc * B + b) * n_dir + DIR) * 4 * d + j;
#pragma unroll
        for (int t4 = 0; t4 < 4; ++t4) {
            double sx = 0.0, sy = 0.0;
#pragma unroll
            for (int qq = 0; qq < kScanSub; ++qq) {
                sx += base[(2 * t4) * kScanThreads + qq * 32 + lane];
                sy += base[(2 * t4 + 1) * kScanThreads + qq * 32 + lane];
            }
            *reinterpret_cast<double2*>(pp + (size_t)t4 * d) = make_double2(sx, sy);
        }
    }
}

}  // namespace sru
