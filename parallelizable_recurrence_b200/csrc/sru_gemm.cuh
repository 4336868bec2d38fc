// sru_gemm.cuh -- the projection of Eq. (1) and its gradients on sm_100a.
//
// "When Attention Meets Fast Recurrence" (T. Lei), background section on SRU:
// the three per-step matrix-vector products of all L steps are grouped into one
// product U^T = [W; W'; W''] X^T, the only dense contraction of the layer.
//
// tc_gemm_pair_kernel computes  out[r, c] (+)= sum_k A(r, k) * B(c, k)  on the
// 5th-generation tensor cores: bf16 operands staged by TMA into 128-byte
// swizzled shared memory, tcgen05.mma issued by a single thread into a fp32
// accumulator in tensor memory (TMEM), and an epilogue that reads TMEM with
// tcgen05.ld and sends the output through shared memory with TMA stores.  A
// cluster of two CTAs (two SMs) computes each 256 x 256 output tile with
// tcgen05.mma.cta_group::2; the kernel is persistent (one pair per two SMs
// walking output tiles) and warp specialised:
//   warp 0        TMA producer (one elected lane), P_STAGES-deep smem ring
//   warp 1        TMEM allocator and MMA issuer (one elected lane, pair leader)
//   warps 2..5    epilogue, one TMEM lane quarter each
// Two 128 x 256 fp32 accumulators per CTA (512 TMEM columns) let the epilogue
// of tile i overlap the main loop of tile i+1.
//
// Operand majorness (which index is contiguous in global memory):
//   U  = X  W^T : A = X  (M x K, K-major), B = W (N x K, K-major)
//   dX = dU W   : A = dU (M x N, K-major), B = W read as (K x N): MN-major
//   dW = dU^T X : A = dU read as (N x M): MN-major, B = X read as (K x M): MN-major
// A K-major tile is one TMA box of (64 K, rows); an MN-major tile is boxes of
// (64 rows, 64 K) placed 8 KB apart.
#pragma once

#include "sru_ptx.cuh"

namespace sru {
namespace gemm {

constexpr int BK = 64;           // k per stage: one 128-byte swizzle row of bf16
constexpr int THREADS = 192;
constexpr uint32_t MN_BOX_BYTES = 64 * 64 * 2;  // one (64 x 64) MN-major box
// kOutF32Acc: add onto the existing fp32 output (TMA reduce-add).
enum OutMode : int { kOutBF16 = 0, kOutF32 = 1, kOutF32Acc = 2 };

// Shared-memory matrix descriptor (tcgen05 "smem descriptor"): start address,
// leading- and stride-dimension byte offsets (16-byte units), descriptor
// version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;  // version for sm_100
    d |= 2ull << 61;  // SWIZZLE_128B
    return d;
}

// ---------------------------------------------------------------------------
// A cluster of two CTAs (two SMs) computes one 256 x 256
// output tile with tcgen05.mma.cta_group::2 (M = 256).  Each CTA stages its own
// 128 rows of A and its own 128 columns of B (32 KB per k-block instead of
// 48 KB for a 128 x 256 tile on one SM), and holds its 128 rows of the
// accumulator in its own TMEM.  The pair leader (cluster rank 0) issues the
// MMAs; both CTAs' TMA loads count on the leader's "full" barrier (the
// .cta_group::2 form of the load); the leader's commits arrive on both CTAs'
// "empty" and "accumulator full" barriers (commit with .multicast::cluster);
// both CTAs' epilogue warps release the accumulator on the leader's barrier.
// No TMA load uses cluster multicast.
#ifndef SRU_GEMM_PAIR_STAGES
#define SRU_GEMM_PAIR_STAGES 6
#endif
constexpr int P_BM = 256, P_BN = 256, P_STAGES = SRU_GEMM_PAIR_STAGES;  // per pair (BK as above)
constexpr int P_CM = 128, P_CN = 128;                  // per CTA
constexpr uint32_t P_A_BYTES = P_CM * BK * 2;          // 16 KB
constexpr uint32_t P_B_BYTES = P_CN * BK * 2;          // 16 KB
constexpr uint32_t P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr uint32_t P_TMEM_COLS = 2 * P_BN;             // two 128 x 256 fp32 accumulators per CTA
// Epilogue staging (non-batched launches): each of the 4 epilogue warps owns
// two 4 KB buffers; a chunk of 32 rows x 128 bytes (64 bf16 or 32 fp32 output
// columns) is written there in the TMA swizzle pattern and leaves by one TMA
// store (or TMA reduce-add), so the output goes out as whole lines instead of
// 16-byte pieces of 32 different rows.
constexpr uint32_t P_EPI_BUF = 4096;
constexpr uint32_t P_EPI_BYTES = 4 * 2 * P_EPI_BUF;
constexpr size_t P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + P_EPI_BYTES + 1024 + 256;
static_assert(P_SMEM_BYTES <= 232448, "pair GEMM shared memory");

// Write one row's accumulator columns (r, fp32 bits) into a staging buffer laid
// out as the TMA tensor's box with 128-byte swizzle: each output row is 128 B
// (64 bf16 or 32 fp32 columns), and its 16-byte chunk c sits at chunk
// c ^ (i % 8) of row i, so the 32 rows' stores of one chunk fall in distinct banks.
template <int OUT>
__device__ __forceinline__ void epilogue_stage_row(uint32_t buf, int i, const uint32_t* r) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t dst = buf + (uint32_t)i * 128u + ((uint32_t)(c ^ (i & 7)) << 4);
        if (OUT == kOutBF16) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 two = __floats2bfloat162_rn(__uint_as_float(r[c * 8 + 2 * e]),
                                                           __uint_as_float(r[c * 8 + 2 * e + 1]));
                w[e] = *reinterpret_cast<uint32_t*>(&two);
            }
            st_shared_v4(dst, w[0], w[1], w[2], w[3]);
        } else {
            st_shared_v4(dst, r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
        }
    }
}

// Accumulator columns per staged box: one 128-byte row per output row.
template <int OUT>
struct EpiChunk {
    static constexpr int kCols = OUT == kOutBF16 ? 64 : 32;
};

// Load kCols consecutive accumulator columns of this warp's 32 TMEM lanes.
template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NC]) {
    static_assert(NC == 32 || NC == 64, "columns per load");
    tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    if (NC == 64) tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[NC == 64 ? 32 : 0]));
}

__host__ __device__ constexpr uint32_t idesc_bf16_pair(bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(P_BN >> 3) << 17) | ((uint32_t)(P_BM >> 4) << 24);
}

// Batched form: `batches` independent products of the same shape.  The
// operands' tensor maps are 3-D with the batch index as coordinate bpos_a /
// bpos_b (1 or 2) and the 2-D tile coordinates in the other two, so a box
// lands in shared memory exactly as in the 2-D case; the output leaves the
// same way through a 3-D map (BPO).
template <int BPOS>
__device__ __forceinline__ void tma_load_tile_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                   int z) {
    if (BPOS == 0)
        tma_load_2d_pair(dst, map, bar, x, y);
    else if (BPOS == 1)
        tma_load_3d_pair(dst, map, bar, x, z, y);
    else
        tma_load_3d_pair(dst, map, bar, x, y, z);
}

// map_out: the output as a tensor of the output type that the epilogue's TMA
// stores write, boxes of 32 rows x 128 bytes with 128-byte swizzle: 2-D (N
// columns, M rows) for single products; for batched ones 3-D with the batch
// index at coordinate BPO: 1 = between columns and rows (batch stride below
// the row stride, e.g. time-major rows t B + b), 2 = outermost.
// A work unit of the pair kernel: output tile (tm, tn) of batch z and its
// k-block range [kb_lo, kb_hi).  CAUSAL (batched square products of SRU++'s
// causal attention, tiles of P_BM = P_BN rows):
//   1  scores S = Q K^T: only the tiles on or below the diagonal (tn <= tm);
//      the tiles above it hold only masked entries, which the softmax never reads;
//   2  A = P V (and dQ = dS K): the reduction over s stops at the end of the
//      row tile, past which every probability (gradient) is 0;
//   3  dV = P^T dA (and dK = dS^T Q): output row tile s0.. reduces over
//      t >= s0 only, since P[t][s] = 0 for t < s.
struct PairUnit {
    int z, tm, tn, kb_lo, kb_hi;
    int split;    // k part of a split-K launch (0 otherwise)
    bool reduce;  // add onto the output (a piece of a tile split in two) instead of storing
};
template <int CAUSAL>
__device__ __forceinline__ PairUnit pair_unit(int u, int m_tiles, int n_tiles, int splits, int kblocks, int kper) {
    PairUnit w;
    if (CAUSAL == 1) {
        const int tri = m_tiles * (m_tiles + 1) / 2;
        w.z = u / tri;
        const int t = u % tri;
        int tm = (int)((sqrtf(8.0f * (float)t + 1.0f) - 1.0f) * 0.5f);
        while (tm * (tm + 1) / 2 > t) --tm;
        while ((tm + 1) * (tm + 2) / 2 <= t) ++tm;
        w.tm = tm;
        w.tn = t - tm * (tm + 1) / 2;
        w.kb_lo = 0;
        w.kb_hi = kblocks;
        w.split = 0;
        w.reduce = false;
        return w;
    }
    const int tiles = m_tiles * n_tiles;
    w.z = u / (tiles * splits);
    const int uu = u % (tiles * splits), tile = uu / splits;
    w.tm = tile / n_tiles;
    w.tn = tile % n_tiles;
    w.split = uu % splits;
    w.kb_lo = w.split * kper;
    w.kb_hi = min(kblocks, w.kb_lo + kper);
    if (CAUSAL == 2) w.kb_hi = min(w.kb_hi, ((w.tm + 1) * P_BM + BK - 1) / BK);
    if (CAUSAL == 3) w.kb_lo = max(w.kb_lo, (w.tm * P_BM) / BK);
    w.reduce = false;
    return w;
}

// The i-th work unit of pair p (of P).  Without a tail split (tail_s == 0) the
// units are dealt round-robin: unit p + i P.  With one (fp32 outputs, one
// batch, no K split): the tiles = F P + R fill F whole rounds round-robin, and
// the R tiles of the last, partial round are cut in two k-pieces, [0, s) and
// [s, K), that both add onto an output region zeroed beforehand (0 + a + b
// rounds the same in either order, so the result is deterministic):
//   pair p < R              the long piece [s, K) of tail tile p
//   pair p >= R             the short pieces [0, s) of tail tiles
//                           (p - R) + j (P - R), j = 0, 1, ..., below R
// so each of the P - R pairs past R takes at most q = ceil(R / (P - R)) short
// pieces.  The host takes s = K / (q + 1): the tail then costs q / (q + 1) of
// a round instead of a whole one (a half for q = 1, two thirds for q = 2).
template <int CAUSAL>
__device__ __forceinline__ bool pair_next(int i, int p, int P, int units, int m_tiles, int n_tiles, int splits,
                                          int kblocks, int kper, int tail_s, PairUnit& w) {
    if (tail_s == 0) {
        const int u = p + i * P;
        if (u >= units) return false;
        w = pair_unit<CAUSAL>(u, m_tiles, n_tiles, splits, kblocks, kper);
        return true;
    }
    const int tiles = m_tiles * n_tiles, F = tiles / P, R = tiles % P;
    int tile = -1;
    bool large = false;
    if (i < F) {
        tile = p + i * P;
    } else if (p < R) {
        if (i == F) {
            tile = F * P + p;
            large = true;
        }
    } else {
        const int t = (p - R) + (i - F) * (P - R);  // short piece j = i - F
        if (t < R) tile = F * P + t;
    }
    if (tile < 0) return false;
    w.z = 0;
    w.tm = tile / n_tiles;
    w.tn = tile % n_tiles;
    w.reduce = i >= F;
    w.split = 0;
    w.kb_lo = (i < F || !large) ? 0 : tail_s;
    w.kb_hi = (i < F || large) ? kblocks : tail_s;
    return true;
}

template <bool A_MN, bool B_MN, int OUT, int BPA = 0, int BPB = 0, int CAUSAL = 0, int BPO = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        const __grid_constant__ CUtensorMap map_out, int M, int N, int K, int splits, int batches,
                        int tail_s, int slab_rows) {
    static_assert(((BPA | BPB) == 0) == (BPO == 0), "batched launches store through a 3-D output map");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi = smem + P_STAGES * P_STAGE_BYTES;  // 1024-aligned staging buffers
    uint64_t* full = reinterpret_cast<uint64_t*>(epi + P_EPI_BYTES);
    uint64_t* empty = full + P_STAGES;
    uint64_t* tfull = empty + P_STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile uint32_t* consumed = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = leader
    const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int m_tiles = (M + P_BM - 1) / P_BM, n_tiles = (N + P_BN - 1) / P_BN;
    const int tiles = m_tiles * n_tiles;
    const int kblocks = (K + BK - 1) / BK;
    // work unit u = (tile u / splits, K part u % splits); the host passes splits = 1
    // batch-major, then tile, then K part (causal scores: the lower-triangle tiles only)
    const int units = (CAUSAL == 1 ? m_tiles * (m_tiles + 1) / 2 : tiles * splits) * batches;
    const int kper = (kblocks + splits - 1) / splits;

    if (threadIdx.x == 0) {
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(&full[s], 1);   // leader only: its producer's expect_tx covers both CTAs' bytes
            mbar_init(&empty[s], 1);  // one multicast commit per phase
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);   // one multicast commit per phase
            mbar_init(&tempty[a], 8);  // leader's: 4 epilogue warps of each CTA
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *consumed = 0;
        fence_mbar_init();
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
        tma_prefetch_desc(&map_out);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, P_TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync_all();  // barriers of both CTAs initialised before any remote use
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t leader_full0 = mapa_shared(smem_u32(&full[0]), 0);
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------ producer (both CTAs)
            uint32_t issued = 0;
            int stage = 0;
            uint32_t phase = 0;
            PairUnit w;
            for (int i = 0; !*abort_flag &&
                            pair_next<CAUSAL>(i, pair_id, n_pairs, units, m_tiles, n_tiles, splits, kblocks, kper,
                                              tail_s, w);
                 ++i) {
                const int z = w.z, kb_lo = w.kb_lo, kb_hi = w.kb_hi;
                const int m0 = w.tm * P_BM + (int)rank * P_CM;
                const int n0 = w.tn * P_BN + (int)rank * P_CN;
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, kErrTimeoutMma) || *abort_flag) {
                        *abort_flag = 1;
                        break;
                    }
                    uint8_t* a_dst = smem + stage * P_STAGE_BYTES;
                    uint8_t* b_dst = a_dst + P_A_BYTES;
                    const int k0 = kb * BK;
                    const uint32_t bar = leader_full0 + (uint32_t)stage * 8u;
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * P_STAGE_BYTES);
                    if (!A_MN) {
                        tma_load_tile_pair<BPA>(a_dst, &map_a, bar, k0, m0, z);
                    } else {
                        tma_load_tile_pair<BPA>(a_dst, &map_a, bar, m0, k0, z);
                        tma_load_tile_pair<BPA>(a_dst + MN_BOX_BYTES, &map_a, bar, m0 + 64, k0, z);
                    }
                    if (!B_MN) {
                        tma_load_tile_pair<BPB>(b_dst, &map_b, bar, k0, n0, z);
                    } else {
                        tma_load_tile_pair<BPB>(b_dst, &map_b, bar, n0, k0, z);
                        tma_load_tile_pair<BPB>(b_dst + MN_BOX_BYTES, &map_b, bar, n0 + 64, k0, z);
                    }
                    ++issued;
                    if (++stage == P_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag && rank == 0) {
                for (uint32_t q = *consumed; q < issued; ++q)
                    mbar_wait(&full[q % P_STAGES], (q / P_STAGES) & 1u, kErrTimeoutLoad);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------------ MMA issuer (leader)
            constexpr uint32_t idesc = idesc_bf16_pair(A_MN, B_MN);
            int stage = 0;
            uint32_t phase = 0, nconsumed = 0;
            int it = 0;
            PairUnit w;
            for (int i = 0; !*abort_flag &&
                            pair_next<CAUSAL>(i, pair_id, n_pairs, units, m_tiles, n_tiles, splits, kblocks, kper,
                                              tail_s, w);
                 ++i, ++it) {
                const int kb_lo = w.kb_lo, kb_hi = w.kb_hi;
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, kErrTimeoutEpilogue)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + acc * P_BN;
                bool ok = true;
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!mbar_wait(&full[stage], phase, kErrTimeoutLoad)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(smem + stage * P_STAGE_BYTES);
                    const uint32_t b_addr = a_addr + P_A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = A_MN ? smem_desc_sw128(a_addr + kk * 2048, MN_BOX_BYTES, 1024)
                                                    : smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = B_MN ? smem_desc_sw128(b_addr + kk * 2048, MN_BOX_BYTES, 1024)
                                                    : smem_desc_sw128(b_addr + kk * 32, 16, 1024);
                        tc_mma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb != kb_lo || kk != 0) ? 1u : 0u);
                    }
                    tc_commit_pair_mc(&empty[stage], 0x3);  // frees this stage in both CTAs
                    *consumed = ++nconsumed;
                    if (++stage == P_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                tc_commit_pair_mc(&tfull[acc], 0x3);  // accumulator ready in both CTAs
            }
            tc_commit_pair_mc(drain, 0x1);
            mbar_wait(drain, 0, kErrTimeoutMma);
        }
    } else {
        // ---------------------------------------------------------- epilogue (both CTAs)
        const int quarter = warp & 3;
        int it = 0;
        uint32_t nstaged = 0;  // chunks this warp has handed to TMA stores
        PairUnit w;
        for (int i = 0; pair_next<CAUSAL>(i, pair_id, n_pairs, units, m_tiles, n_tiles, splits, kblocks, kper, tail_s, w);
             ++i, ++it) {
            const int z = w.z;
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            const int m0 = w.tm * P_BM + (int)rank * P_CM, n0 = w.tn * P_BN;
            const bool ok = mbar_wait(&tfull[acc], acc_phase, kErrTimeoutMma);
            if (!__all_sync(0xffffffffu, ok) || *abort_flag) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after_sync();
            // the accumulator leaves in chunks of kCols columns; the TMEM load of chunk
            // g + 1 is issued before chunk g is converted and stored, so its latency
            // overlaps that work
            constexpr int NC = EpiChunk<OUT>::kCols, NG = P_BN / NC;
            const int ng = min(NG, (N - n0 + NC - 1) / NC);  // chunks that start inside N (>= 1)
            const uint32_t tacc = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * P_BN;
            uint32_t r0[NC], r1[NC];
            tmem_ld_cols<NC>(tacc, r0);
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                if (g >= ng) break;  // uniform across the warp
                uint32_t(&cur)[NC] = (g & 1) ? r1 : r0;
                uint32_t(&nxt)[NC] = (g & 1) ? r0 : r1;
                tc_wait_ld();  // chunk g (and nothing else) is in flight
                if (g + 1 < ng) tmem_ld_cols<NC>(tacc + (g + 1) * NC, nxt);
                const int col0 = n0 + g * NC;
                // buffer (nstaged & 1) was last read by the store issued two chunks ago
                const uint32_t buf = smem_u32(epi) + (uint32_t)(quarter * 2 + (nstaged & 1)) * P_EPI_BUF;
                if (nstaged >= 2) {
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                }
                epilogue_stage_row<OUT>(buf, lane, cur);
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    const void* src = epi + (size_t)(quarter * 2 + (nstaged & 1)) * P_EPI_BUF;
                    // split-K: k part s lands in slab s, rows s * slab_rows ..
                    const int orow = m0 + quarter * 32 + w.split * slab_rows;
                    if (BPO == 0) {
                        if (OUT == kOutF32Acc || w.reduce)
                            tma_reduce_add_2d(&map_out, src, col0, orow);
                        else
                            tma_store_2d(&map_out, src, col0, orow);
                    } else if (OUT == kOutF32Acc) {
                        if (BPO == 1) tma_reduce_add_3d(&map_out, src, col0, z, orow);
                        else tma_reduce_add_3d(&map_out, src, col0, orow, z);
                    } else {
                        if (BPO == 1) tma_store_3d(&map_out, src, col0, z, orow);
                        else tma_store_3d(&map_out, src, col0, orow, z);
                    }
                    bulk_commit_group();
                }
                ++nstaged;
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty0 + (uint32_t)acc * 8u);
        }
        if (lane == 0) bulk_wait_group<0>();  // every store of this warp has landed
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, P_TMEM_COLS);
    }
}

// Zero the output regions of the tail tiles (tiles first_tile .. first_tile +
// gridDim.x - 1 of P_BM x P_BN, clipped to R x C, row stride ldo floats) that
// the tail split's two pieces then add onto; P_BM / kZeroRows blocks per tile.
// Block (x, y): tile first_tile + x, rows y * kZeroRows .. of it.
constexpr int kZeroRows = 16;
__global__ void __launch_bounds__(256) zero_tail_tiles_kernel(float* __restrict__ out, int R, int C, long long ldo,
                                                              int n_tiles, int first_tile) {
    const int tile = first_tile + blockIdx.x;
    const int r0 = (tile / n_tiles) * P_BM + blockIdx.y * kZeroRows, c0 = (tile % n_tiles) * P_BN;
    const int rows = min(kZeroRows, R - r0), cols = min(P_BN, C - c0);  // C % 8 == 0: cols a multiple of 4
    for (int e = threadIdx.x; e < rows * (cols / 4); e += blockDim.x) {
        const int r = e / (cols / 4), c4 = e % (cols / 4);
        *reinterpret_cast<float4*>(out + (size_t)(r0 + r) * ldo + c0 + 4 * c4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// Split-K: out[r][c] = sum over s = 0, 1, .. of slabs[s * slab_rows + r][c], in
// that order (the same bits every run); four columns per thread (C % 4 == 0).
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4* __restrict__ slabs, float4* __restrict__ out,
                                                            int R, int C4, int slab_rows, int splits) {
    const size_t n = (size_t)R * C4;
    for (size_t e = blockIdx.x * (size_t)256 + threadIdx.x; e < n; e += (size_t)gridDim.x * 256) {
        const size_t r = e / C4, c = e % C4;
        float4 acc = slabs[r * C4 + c];
        for (int sp = 1; sp < splits; ++sp) {
            const float4 v = slabs[((size_t)sp * slab_rows + r) * C4 + c];
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        out[e] = acc;
    }
}

// ---------------------------------------------------------------------------
// CUDA-core fp32 product with explicit element strides (the fp32 path):
//   out[r * ldo + c] (+)= sum_k A[r*a_rs + k*a_ks] * B[c*b_rs + k*b_ks]
// 64 x 64 output tile per 256-thread CTA, 4 x 4 outputs per thread.
constexpr int ST = 64, SK = 16;

__global__ void __launch_bounds__(256)
    simt_gemm_f32_kernel(const float* __restrict__ A, long long a_rs, long long a_ks, const float* __restrict__ Bm,
                         long long b_rs, long long b_ks, float* __restrict__ out, long long ldo, int R, int C, int K,
                         int accumulate) {
    __shared__ float As[SK][ST + 1];
    __shared__ float Bs[SK][ST + 1];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int r0 = blockIdx.y * ST, c0 = blockIdx.x * ST;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += SK) {
        for (int e = threadIdx.x; e < SK * ST; e += 256) {
            const int kk = e / ST, rr = e % ST;
            const int k = k0 + kk;
            As[kk][rr] = (r0 + rr < R && k < K) ? A[(long long)(r0 + rr) * a_rs + (long long)k * a_ks] : 0.f;
            Bs[kk][rr] = (c0 + rr < C && k < K) ? Bm[(long long)(c0 + rr) * b_rs + (long long)k * b_ks] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < SK; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                bb[i] = Bs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i], bb[jj], acc[i][jj]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int r = r0 + ty * 4 + i, c = c0 + tx * 4 + jj;
            if (r < R && c < C) {
                float* o = out + (long long)r * ldo + c;
                *o = accumulate ? *o + acc[i][jj] : acc[i][jj];
            }
        }
}

}  // namespace gemm
}  // namespace sru
