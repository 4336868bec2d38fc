// sru_fused.cuh -- the projection of Eq. (1) and the recurrence of Eqs. (2)-(5)
// in one kernel: "When Attention Meets Fast Recurrence" (T. Lei), Figure 2(a),
// whose two boxes (the grouped matrix multiplication, then the element-wise
// recurrence) run here as the main loop and the epilogue of one persistent
// tcgen05 kernel, so the projection output U never has to be read back from
// HBM (and is not written at all when no backward follows).
//
// Work item = (time tile of kTt steps, direction, pair of batch groups, 64
// channels).  A CTA pair (cluster of two SMs) computes, with
// tcgen05.mma.cta_group::2 (M = 256, N = 192),
//     D[(t, b), (half, gate, c)] = sum_k X[t*B + b, k] * W_cat[dir, gate, j0 + 32 half + c, k]
// where each CTA owns the kTt x kBb = 128 (t, b) rows of its batch group (its
// A operand: one 3-D TMA box (64 k, kBb rows, kTt steps) of X) and supplies
// half of the 192 W_cat rows (one 3-D box (64 k, 32 channels, 3 gates)).
// Each CTA's accumulator rows are its own 128 (t, b) rows, all 192 columns,
// i.e. every gate of the item's 64 channels for its 4 batch rows.
//
// Epilogue (4 warps per CTA): the accumulator is read from TMEM (thread =
// one (t, b) row), rounded to bf16 -- the storage type of U on the unfused
// path -- and written to a shared-memory U tile [t][b][gate][64 ch] in the
// 128-byte TMA swizzle (conflict-free both ways).  Where the caller wants U
// (training), one TMA store sends that tile to global memory.  Then each warp
// walks Eqs. (2)-(5) for one batch row over the tile's kTt steps in the
// direction's time order, one thread per channel pair with the same packed
// fp32x2 cell as the sequential kernels (so h equals sru_forward's on the
// same bf16 U, bit for bit), writing h, the 16-step state checkpoints the
// backward reads, and c_T.
//
// Time tiles of one (batch row, direction, channel slice) stream are walked
// in order but may run on different CTAs: items are dealt round-robin in
// (time tile, stream) order, and the state leaving a tile is handed to the
// next through one 64-bit word per channel holding the state and the number
// of the tile that wrote it (tile + 1; the words are zeroed before the
// launch).  An aligned 64-bit access is single-copy atomic, so the reader
// that sees its predecessor's tile number in a word has that tile's state in
// the same word: no flag, fence or second round trip.  The MMAs of every item
// run without waiting; only the epilogue's walk waits for its predecessor's
// carry, which was dealt earlier.  Every CTA of the grid must be resident
// (one per SM, grid <= SM count); waits are bounded (2 s) so that a GPU
// shared with other work cannot hang the kernel.
#pragma once

#include "sru_recurrence.cuh"
#include "sru_scan.cuh"

namespace sru {
namespace fused {

constexpr int kTt = 32;                  // time steps per tile (a warp-wide row-validity ballot)
constexpr int kBb = 4;                   // batch rows per CTA (one epilogue warp each)
constexpr int kCh = 64;                  // channels per item
constexpr int kRows = kTt * kBb;         // 128 accumulator rows per CTA
constexpr int kN = 3 * kCh;              // 192 accumulator columns
constexpr int kBK = 64;                  // k per stage (one 128-byte swizzle row)
constexpr uint32_t kABytes = kRows * kBK * 2;          // 16 KB of X per CTA
constexpr uint32_t kBBytes = (kN / 2) * kBK * 2;       // 12 KB of W_cat per CTA and slice
constexpr uint32_t kUTileBytes = kRows * 3 * 128;      // 48 KB per slice: [t][b][gate] lines of 64 bf16
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;                      // column stride of accumulators
constexpr int kThreads = 192;
static_assert(kTt == 32, "one ballot covers a tile's rows");
static_assert(kTt % kChunkT == 0, "checkpoint interval divides the tile");

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B (both
// K-major), N = 192, M = 256 (cta_group::2).
__host__ __device__ constexpr uint32_t idesc_fused() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(16u >> 4) << 16;     // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024u >> 4) << 32;   // 8 rows x 128 B between core-matrix groups
    d |= 1ull << 46;                     // sm_100 descriptor version
    d |= 2ull << 61;                     // 128-byte swizzle
    return d;
}

// Named barrier / barrier-reduction over the 4 epilogue warps (barrier 1).
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool epi_sync_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, const void* src, int c0, int c1, int c2, int c3,
                                             int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}

// Tagged carry words of a channel pair: (tag << 32) | float bits, one 16-byte
// access of two single-copy-atomic 64-bit elements.
__device__ __forceinline__ void ld_carry2(const unsigned long long* p, unsigned& tag0, unsigned& tag1, float2& c) {
    unsigned long long w0, w1;
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
    tag0 = (unsigned)(w0 >> 32);
    tag1 = (unsigned)(w1 >> 32);
    c = make_float2(__uint_as_float((unsigned)w0), __uint_as_float((unsigned)w1));
}
__device__ __forceinline__ void st_carry2(unsigned long long* p, unsigned tag, float2 c) {
    const unsigned long long hi = (unsigned long long)tag << 32;
    const unsigned long long w0 = hi | __float_as_uint(c.x), w1 = hi | __float_as_uint(c.y);
    asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(w0), "l"(w1) : "memory");
}

// Shared-memory address of the 32-bit word holding channels (2l, 2l+1) of
// gate g at accumulator row r in the swizzled U tile.
__device__ __forceinline__ uint32_t utile_word(uint32_t utile, int r, int g, int l) {
    const uint32_t line = (uint32_t)(r * 3 + g);
    return utile + line * 128u + ((((uint32_t)l >> 2) ^ (line & 7u)) << 4) + ((uint32_t)l & 3u) * 4u;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

struct FusedArgs {
    const float* x;        // (L, B, d) fp32 highway input
    const float* v;        // (n_dir, 2, d)
    const float* bias;     // (n_dir, 2, d)
    const float* c0;       // (B, n_dir, d) or null
    const uint8_t* mask;   // (L, B) or null
    float* h;              // (L, B, n_dir, d)
    float* c_T;            // (B, n_dir, d)
    float* ckpt;           // (ceil(L/16), B, n_dir, d) or null
    unsigned long long* carry;  // (B, n_dir, d): (tile + 1) << 32 | state bits, from a tile to the next
                                //  (zeroed before the launch)
    int L, B, d, n_dir;
    float alpha;
    int write_u;           // store the U tile with map_u
};

// x of one tile half (rows i0 .. i0+15, those before L), for one thread's
// channel pair; loaded ahead of use so that its latency is off the chain.
__device__ __forceinline__ void load_x_half(float2 (&wx)[kChunkT], const float* __restrict__ xp, int i0, int nrows,
                                            size_t tstride_x, bool jok) {
#pragma unroll
    for (int i = 0; i < kChunkT; ++i)
        wx[i] = (jok && i0 + i < nrows) ? load_pair(xp + (size_t)(i0 + i) * tstride_x) : f2(0.f);
}

// Walk kChunkT steps of one tile half (rows i0 .. i0+15 of the tile in time
// order, visited in the direction's order) for one thread's channel pair,
// with the half's x already in registers.
// word(r, g): shared-memory address of this thread's bf16 pair of gate g at
// accumulator row r (the U tile's layout is the caller's).
template <int DIR, typename WordAddr>
__device__ __forceinline__ float2 fused_chunk(WordAddr word, int q, int i0, uint32_t valid16, float2 c,
                                              const GateParams2& p, float2 alpha2, const float2 (&wx)[kChunkT],
                                              float* __restrict__ hp, size_t tstride_h, bool jok, int nrows) {
    constexpr uint32_t kFull = (1u << kChunkT) - 1u;
    if (valid16 == kFull) {
        uint32_t wc[kChunkT], wf[kChunkT], wr[kChunkT];
#pragma unroll
        for (int i = 0; i < kChunkT; ++i) {
            const int r = (i0 + i) * kBb + q;
            wc[i] = lds_u32(word(r, 0));
            wf[i] = lds_u32(word(r, 1));
            wr[i] = lds_u32(word(r, 2));
        }
        // pass 1: the state chain (forget gate and c only); pass 2: reset gate and h
        float2 cprev[kChunkT], cs[kChunkT];
#pragma unroll
        for (int s = 0; s < kChunkT; ++s) {
            const int i = DIR == 0 ? s : kChunkT - 1 - s;
            cprev[i] = c;
            const float2 uc = bf16x2_to_float2(wc[i]);
            c = fma2(sru_forget2(c, bf16x2_to_float2(wf[i]), p), sub2(c, uc), uc);  // Eq. (4)
            cs[i] = c;
        }
        float2 hv[kChunkT];
#pragma unroll
        for (int i = 0; i < kChunkT; ++i) {
            const float2 r = sru_reset2(cprev[i], bf16x2_to_float2(wr[i]), p);
            const float2 ax = mul2(alpha2, wx[i]);
            hv[i] = fma2(r, sub2(cs[i], ax), ax);  // Eq. (5)
        }
        if (jok) {
#pragma unroll
            for (int i = 0; i < kChunkT; ++i) store_pair(hp + (size_t)(i0 + i) * tstride_h, hv[i]);
        }
        return c;
    }
#pragma unroll
    for (int s = 0; s < kChunkT; ++s) {
        const int i = DIR == 0 ? s : kChunkT - 1 - s;
        if (i0 + i >= nrows) continue;  // beyond L
        float2 hv = f2(0.f);
        if ((valid16 >> i) & 1u) {
            const int r = (i0 + i) * kBb + q;
            float2 f, rr;
            c = sru_cell2(c, bf16x2_to_float2(lds_u32(word(r, 0))), bf16x2_to_float2(lds_u32(word(r, 1))),
                          bf16x2_to_float2(lds_u32(word(r, 2))), p, f, rr);
            const float2 ax = mul2(alpha2, wx[i]);
            hv = fma2(rr, sub2(c, ax), ax);
        }
        if (jok) store_pair(hp + (size_t)(i0 + i) * tstride_h, hv);
    }
    return c;
}

constexpr int kStages = 6;
constexpr uint32_t kStageBytes = kABytes + kBBytes;  // 28 KB: X tile + this CTA's half of the W_cat rows
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + kUTileBytes + 1024 + 256;
static_assert(kSmemBytes <= 232448, "fused kernel shared memory");

// map_x: X as 3-D (d, B, L) bf16, box (64, kBb, kTt), 128-byte swizzle.
// map_w: W_cat as 3-D (d, d, n_dir*3) bf16, box (64, 32, 3), 128-byte swizzle.
// map_u: U as 5-D (d, 3, n_dir, B, L) bf16, box (64, 3, 1, kBb, kTt), 128-byte
//        swizzle (only used when a.write_u).
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sru_fused_fwd_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                         const __grid_constant__ CUtensorMap map_u, const FusedArgs a) {
    constexpr int kAccBufs = 2;  // accumulators in flight
    constexpr int NS = 1;        // 64-channel slices per work item (the loops below take any count; one measured fastest)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* utile_p = smem + kStages * kStageBytes;  // 1024-aligned U tile(s)
    uint64_t* full = reinterpret_cast<uint64_t*>(utile_p + NS * kUTileBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + kAccBufs;
    uint64_t* drain = tempty + kAccBufs;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile uint32_t* consumed = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = leader
    const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int L = a.L, B = a.B, d = a.d, n_dir = a.n_dir;
    const int nT = (L + kTt - 1) / kTt;                     // time tiles
    const int njs = (d + kCh - 1) / kCh;                    // channel slices
    const int njg = (njs + NS - 1) / NS;                    // groups of NS slices (one item each)
    const int nbgp = (B + 2 * kBb - 1) / (2 * kBb);         // pairs of batch groups
    const int streams = n_dir * nbgp * njg;
    const int items = nT * streams;
    const int kblocks = (d + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int acc = 0; acc < kAccBufs; ++acc) {
            mbar_init(&tfull[acc], 1);
            mbar_init(&tempty[acc], 8);  // leader's: the 4 epilogue warps of each CTA
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *consumed = 0;
        fence_mbar_init();
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
        if (a.write_u) tma_prefetch_desc(&map_u);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync_all();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t leader_full0 = mapa_shared(smem_u32(&full[0]), 0);
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);

    // item u -> (walk-order time tile, direction, batch-group pair, slice group)
    auto decode = [&](int u, int& tt, int& dir, int& bgp, int& jg) {
        tt = u / streams;
        int s = u % streams;
        jg = s % njg;
        s /= njg;
        bgp = s % nbgp;
        dir = s / nbgp;
    };
    // accumulator of buffer acc, slice s: TMEM columns from (acc + s) * kAccCols
    // (one of acc, s is always 0)

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------ producer (both CTAs)
            uint32_t issued = 0;
            int stage = 0;
            uint32_t phase = 0;
            for (int u = pair_id; u < items && !*abort_flag; u += n_pairs) {
                int tt, dir, bgp, jg;
                decode(u, tt, dir, bgp, jg);
                const int tp = dir == 0 ? tt : nT - 1 - tt;
                const int b0 = bgp * 2 * kBb + (int)rank * kBb;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, kErrTimeoutMma) || *abort_flag) {
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* a_dst = smem + stage * kStageBytes;
                    const uint32_t bar = leader_full0 + (uint32_t)stage * 8u;
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
                    tma_load_3d_pair(a_dst, &map_x, bar, kb * kBK, b0, tp * kTt);
#pragma unroll
                    for (int s = 0; s < NS; ++s)
                        tma_load_3d_pair(a_dst + kABytes + s * kBBytes, &map_w, bar, kb * kBK,
                                         (jg * NS + s) * kCh + (int)rank * (kCh / 2), dir * 3);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag && rank == 0) {
                for (uint32_t qd = *consumed; qd < issued; ++qd)
                    mbar_wait(&full[qd % kStages], (qd / kStages) & 1u, kErrTimeoutLoad);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------------ MMA issuer (leader)
            constexpr uint32_t idesc = idesc_fused();
            int stage = 0;
            uint32_t phase = 0, nconsumed = 0;
            int it = 0;
            for (int u = pair_id; u < items && !*abort_flag; u += n_pairs, ++it) {
                const int acc = it % kAccBufs;
                const uint32_t acc_phase = (it / kAccBufs) & 1;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, kErrTimeoutEpilogue)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, kErrTimeoutLoad)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
                        for (int s = 0; s < NS; ++s)
                            tc_mma_bf16_pair(tmem_base + (uint32_t)(acc + s) * kAccCols, sdesc_sw128(a_addr + kk * 32),
                                             sdesc_sw128(a_addr + kABytes + s * kBBytes + kk * 32), idesc,
                                             (kb | kk) != 0 ? 1u : 0u);
                    tc_commit_pair_mc(&empty[stage], 0x3);
                    *consumed = ++nconsumed;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                tc_commit_pair_mc(&tfull[acc], 0x3);
            }
            tc_commit_pair_mc(drain, 0x1);
            mbar_wait(drain, 0, kErrTimeoutMma);
        }
    } else {
        // ---------------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;  // TMEM lane quarter = this warp's batch row in the group
        const uint32_t utile0 = smem_u32(utile_p);
        const bool issuer = warp == 2 && lane == 0;  // sends the U tiles by TMA
        const int cj = 2 * lane;
        const float2 alpha2 = f2(a.alpha);
        const size_t tstride_x = (size_t)B * d;
        const size_t tstride_h = (size_t)B * n_dir * d;
        const int nch = (L + kChunkT - 1) / kChunkT;
        int it = 0;
        bool stored = false;
        for (int u = pair_id; u < items; u += n_pairs, ++it) {
            int tt, dir, bgp, jg;
            decode(u, tt, dir, bgp, jg);
            const int tp = dir == 0 ? tt : nT - 1 - tt;
            const int acc = it % kAccBufs;
            const uint32_t acc_phase = (it / kAccBufs) & 1;
            const bool ok = mbar_wait(&tfull[acc], acc_phase, kErrTimeoutMma);
            // the previous item's U stores must be done reading the tiles before they are rewritten
            if (issuer && stored) bulk_wait_group_read<0>();
            if (epi_sync_or(!__all_sync(0xffffffffu, ok) || *abort_flag)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            // ---- this warp's streams: batch row b, channel pair (j, j+1) of each slice.
            // What the first slice's walk reads from global memory is requested now, so
            // that its latency passes under the accumulator transpose below.
            const int b0 = bgp * 2 * kBb + (int)rank * kBb;
            const int b = b0 + q;
            const bool brow = b < B;
            const int bd = b * n_dir + dir;
            const int t_base = tp * kTt;
            const int nrows = min(kTt, L - t_base);
            const int i_first = dir == 0 ? 0 : kTt - kChunkT;  // first tile half in walk order
            const int i_second = kTt - kChunkT - i_first;
            float2 xa[kChunkT];
            GateParams2 p;
            float2 c;
            bool have;
            int j;
            bool jok;
            // x of the first half, gate parameters and entering state of slice s
            auto prefetch = [&](int s) {
                j = (jg * NS + s) * kCh + cj;
                jok = brow && j < d;
                load_x_half(xa, a.x + (size_t)t_base * tstride_x + (size_t)b * d + j, i_first, nrows, tstride_x, jok);
                p = make_gate_params2(f2(0.f), f2(0.f), f2(0.f), f2(0.f));
                c = f2(0.f);
                have = true;
                if (jok) {
                    p = make_gate_params2(load_pair(a.v + (dir * 2 + 0) * d + j), load_pair(a.v + (dir * 2 + 1) * d + j),
                                          load_pair(a.bias + (dir * 2 + 0) * d + j),
                                          load_pair(a.bias + (dir * 2 + 1) * d + j));
                    if (tt == 0) {
                        if (a.c0 != nullptr) c = load_pair(a.c0 + (size_t)bd * d + j);
                    } else {
                        unsigned g0, g1;
                        ld_carry2(a.carry + (size_t)bd * d + j, g0, g1, c);
                        have = g0 == (unsigned)tt && g1 == (unsigned)tt;  // written by tile tt - 1
                    }
                }
            };
            prefetch(0);
            // rows of this tile that exist (t < L) and are not padded, bit i = step t_base + i
            bool vrow = brow && lane < nrows;
            if (vrow && a.mask != nullptr) vrow = a.mask[(size_t)(t_base + lane) * B + b] == 0;
            const uint32_t valid = __ballot_sync(0xffffffffu, vrow);
            // ---- accumulator rows (t, b) -> bf16 U tiles, 128-byte swizzled lines [t][b][gate]
            {
                const int r = q * 32 + lane;
#pragma unroll 1
                for (int c2 = 0; c2 < 3 * NS; ++c2) {
                    const int s = c2 / 3;
                    uint32_t v[2][32];
                    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc + s) * kAccCols +
                                           (c2 % 3) * 64;
                    tmem_ld_32x32b_x32(taddr, v[0]);
                    tmem_ld_32x32b_x32(taddr + 32, v[1]);
                    tc_wait_ld();
                    const uint32_t utile = utile0 + (uint32_t)s * kUTileBytes;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int c6 = 2 * (c2 % 3) + k;
                        const int half = c6 / 3, g = c6 % 3;
                        const uint32_t line = (uint32_t)(r * 3 + g);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint32_t w[4];
#pragma unroll
                            for (int k2 = 0; k2 < 4; ++k2) {
                                __nv_bfloat162 two = __floats2bfloat162_rn(__uint_as_float(v[k][e * 8 + 2 * k2]),
                                                                           __uint_as_float(v[k][e * 8 + 2 * k2 + 1]));
                                w[k2] = *reinterpret_cast<uint32_t*>(&two);
                            }
                            const uint32_t chunk = (uint32_t)(half * 4 + e);
                            st_shared_v4(utile + line * 128u + ((chunk ^ (line & 7u)) << 4), w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty0 + (uint32_t)acc * 8u);  // accumulator free
            fence_proxy_async_shared();  // the tiles' writes, visible to the TMA store
            epi_sync();
            if (issuer && a.write_u && b0 < B) {  // (a group wholly beyond B has no rows to store)
#pragma unroll
                for (int s = 0; s < NS; ++s)
                    if ((jg * NS + s) < njs)
                        tma_store_5d(&map_u, utile_p + s * kUTileBytes, (jg * NS + s) * kCh, 0, dir, b0, t_base);
                bulk_commit_group();
                stored = true;
            }
            if (!brow) continue;
            // ---- Eqs. (2)-(5) over the tile's steps in the direction's order, slice by slice
#pragma unroll 1
            for (int s = 0; s < NS; ++s) {
                if (s > 0) prefetch(s);
                if ((jg * NS + s) >= njs) break;  // a slice wholly beyond d
                unsigned long long* cw = a.carry + (size_t)bd * d + j;  // this pair's carry words
                if (!have) {
                    // the previous tile of this stream has not handed over yet: re-read (bounded)
                    const uint64_t t0 = globaltimer_ns();
                    for (;;) {
                        unsigned g0, g1;
                        ld_carry2(cw, g0, g1, c);
                        if (g0 == (unsigned)tt && g1 == (unsigned)tt) break;
                        if (*reinterpret_cast<volatile unsigned*>(&g_error_word) != 0u) break;
                        if (globaltimer_ns() - t0 > kWaitLimitNs) {
                            record_error(kErrTimeoutScan);
                            break;
                        }
                    }
                }
                const uint32_t utile = utile0 + (uint32_t)s * kUTileBytes;
                const float* xp = a.x + (size_t)t_base * tstride_x + (size_t)b * d + j;
                float* hp = a.h + (size_t)t_base * tstride_h + (size_t)bd * d + j;
                float2 xb[kChunkT];
                load_x_half(xb, xp, i_second, nrows, tstride_x, jok);  // under the first half's walk
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i0 = hh == 0 ? i_first : i_second;
                    const int tc = (t_base + i0) / kChunkT;
                    if (tc >= nch) continue;  // wholly beyond L
                    if (a.ckpt != nullptr && jok) store_pair(a.ckpt + ((size_t)tc * B * n_dir + bd) * d + j, c);
                    const uint32_t v16 = (valid >> i0) & ((1u << kChunkT) - 1u);
                    auto word = [&](int r, int g) { return utile_word(utile, r, g, lane); };
                    if (dir == 0)
                        c = fused_chunk<0>(word, q, i0, v16, c, p, alpha2, hh == 0 ? xa : xb, hp, tstride_h, jok, nrows);
                    else
                        c = fused_chunk<1>(word, q, i0, v16, c, p, alpha2, hh == 0 ? xa : xb, hp, tstride_h, jok, nrows);
                }
                if (tt + 1 < nT) {
                    if (jok) st_carry2(cw, (unsigned)(tt + 1), c);
                } else if (jok) {
                    store_pair(a.c_T + (size_t)bd * d + j, c);
                }
            }
        }
        if (issuer && stored) bulk_wait_group<0>();  // every U store has landed
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace fused
}  // namespace sru
