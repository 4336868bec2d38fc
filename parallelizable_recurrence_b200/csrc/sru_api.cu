// sru_api.cu -- the C ABI of libsru.so (declared in include/sru.h): argument
// validation, TMA tensor-map construction and kernel dispatch.  The library is
// built as this single translation unit so the device error word has one
// definition; the kernels live in the included .cuh files.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/sru.h"
#include "sru_gemm.cuh"
#include "sru_recurrence.cuh"
#include "sru_attention.cuh"
#include "sru_decode.cuh"
#include "sru_scan.cuh"
#include "sru_fused.cuh"

namespace {

thread_local int g_last_cuda_error = 0;

sru_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return SRU_ERR_CUDA;
}

#define SRU_CUDA_TRY(expr)                          \
    do {                                            \
        cudaError_t e_ = (expr);                    \
        if (e_ != cudaSuccess) return cuda_fail(e_); \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// the per-channel vectors (v, b, c0, c_T and their gradients) are read and
// written as 8-byte channel pairs; a null (optional) pointer passes
inline bool aligned8_or_null(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// rank-R tiled map; dims/box innermost first; strides (bytes) of dims 1..R-1
#ifndef SRU_TMA_L2_PROMOTION
#define SRU_TMA_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                    reinterpret_cast<const cuuint64_t*>(strides), reinterpret_cast<const cuuint32_t*>(box), estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, SRU_TMA_L2_PROMOTION,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------- device facts
constexpr int kMaxDevices = 64;

bool no_device = false;  // CUDA unavailable: do not retry its (slow) initialisation

int sm_count() {
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    if (no_device) return 148;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        if (cudaGetLastError() == cudaErrorNoDevice || dev < 0) no_device = true;
        return 148;
    }
    if (cache[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 148;
    }
    return cache[dev];
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_smem(const void* kernel, size_t bytes) {
    static std::mutex mu;
    static const void* done_kernel[256];
    static int done_dev[256];
    static int ndone = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < ndone; ++i)
        if (done_kernel[i] == kernel && done_dev[i] == dev) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    if (ndone < 256) {
        done_kernel[ndone] = kernel;
        done_dev[ndone] = dev;
        ++ndone;
    }
    return cudaSuccess;
}

// ---------------------------------------------------------- workspace layout
// [checkpoints | fused-forward carry words | launch order | dv/db partial sums | scan
//  flags | scan aggregates A, B, prefix].  The scan regions exist only when a
// scan can run (see ws_has_scan); the offsets of the first two regions do not
// depend on the flags.
struct WsLayout {
    size_t ckpt_off, carry_off, order_off, partial_off, flags_off, agg_a_off, agg_b_off, prefix_off, total;
    int64_t scan_items;
};

int64_t scan_chunks(int64_t L) { return (L + sru::kScanT - 1) / sru::kScanT; }

bool ws_has_scan(unsigned flags, int64_t L, int64_t B, int64_t d, int n_dir);

WsLayout ws_layout(int64_t L, int64_t B, int64_t d, int n_dir, unsigned flags) {
    WsLayout w{};
    const int64_t nch = (L + sru::kChunkT - 1) / sru::kChunkT;
    const int64_t n_jt = (d + sru::kRecCJ - 1) / sru::kRecCJ;
    const bool scan = ws_has_scan(flags, L, B, d, n_dir);
    size_t off = 0;
    w.ckpt_off = off;
    off += round256((size_t)nch * B * n_dir * d * sizeof(float));
    w.carry_off = off;
    off += round256((size_t)B * n_dir * d * sizeof(unsigned long long));
    w.order_off = off;
    off += round256((size_t)B * n_dir * sizeof(int));
    w.partial_off = off;
    const int64_t partial_rows = scan ? scan_chunks(L) * B : B;
    off += round256((size_t)partial_rows * n_dir * 4 * d * sizeof(double));
    w.scan_items = scan ? scan_chunks(L) * n_jt * B * n_dir : 0;
    w.flags_off = off;
    if (scan) {
        off += round256((size_t)(w.scan_items + 1) * sizeof(unsigned));
        w.agg_a_off = off;
        off += round256((size_t)w.scan_items * sru::kRecCJ * sizeof(float));
        w.agg_b_off = off;
        off += round256((size_t)w.scan_items * sru::kRecCJ * sizeof(float));
        w.prefix_off = off;
        off += round256((size_t)w.scan_items * sru::kRecCJ * sizeof(float));
    }
    w.total = off;
    return w;
}

sru::ScanState scan_state(void* workspace, const WsLayout& w, unsigned flags) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    sru::ScanState ss;
    ss.withhold = (flags & SRU_FLAG_TEST_WITHHOLD_CARRY) ? 0 : -1;
    ss.flags = reinterpret_cast<unsigned*>(ws + w.flags_off);
    ss.agg_a = reinterpret_cast<float*>(ws + w.agg_a_off);
    ss.agg_b = reinterpret_cast<float*>(ws + w.agg_b_off);
    ss.prefix = reinterpret_cast<float*>(ws + w.prefix_off);
    return ss;
}

// ------------------------------------------------ sequential kernel or scan
// The sequential kernels give every CTA a whole sequence (L/16 chunks walked
// one after another); the chunked scans cut time into kScanT-step work items
// at the price of a second pass over each item and a look-back.  Measured on
// B200 over layers from L256 B32 d512 to L8192 B4 d512: one wave of resident
// forward-scan CTAs costs about as much as kScanWaveChunksFwd sequential
// 16-step chunks (about 12 us against 1.5-2 us per chunk), one wave of
// backward-scan CTAs about kScanWaveChunksBwd (about 12-15 us against 2.3-3
// us), so a scan is taken when its waves cost fewer chunks than the sequence
// has.  Only grids that leave SMs idle (fewer than two sequential CTAs per SM)
// are candidates.  The forward scan needs SRU_FLAG_V_ZERO (linear state
// recurrence); the backward scan is exact for any v (the state-gradient
// recurrence is affine).  The FORCE flags override.
constexpr int64_t kScanWaveChunksFwd = 8;
constexpr int64_t kScanWaveChunksBwd = 5;

int64_t seq_ctas(int64_t B, int64_t d, int n_dir_per_launch) {
    return ((d + sru::kRecCJ - 1) / sru::kRecCJ) * B * n_dir_per_launch;
}
bool scan_candidate(int64_t B, int64_t d, int n_dir_per_launch) {
    return seq_ctas(B, d, n_dir_per_launch) < 2 * (int64_t)sm_count();
}
// Scan CTAs (kScanThreads threads, `smem` bytes) resident per SM without a
// device to ask: shared memory bounds it (1 KB per CTA is reserved by the
// system).
int smem_resident(size_t smem) {
    static int cap[kMaxDevices] = {0};
    int dev = 0;
    int bytes = 228 * 1024;
    sm_count();  // sets no_device when CUDA is unavailable
    if (!no_device && cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
        if (cap[dev] == 0) {
            int n = 0;
            cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
            cap[dev] = n > 0 ? n : bytes;
        }
        bytes = cap[dev];
    }
    const int n = (int)(bytes / (smem + 1024));
    return n < 1 ? 1 : (n > 8 ? 8 : n);
}
// A scan kernel's CTAs resident per SM (registers and shared memory), from the
// occupancy calculator; the shared-memory bound when it cannot answer.
int scan_resident(const void* kern, size_t smem) {
    if (no_device || ensure_smem(kern, smem) != cudaSuccess) return smem_resident(smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, sru::kScanThreads, smem) != cudaSuccess || n < 1) {
        cudaGetLastError();
        return smem_resident(smem);
    }
    return n;
}
bool scan_pays(int64_t L, int64_t ctas, int per_sm, int64_t wave_chunks) {
    const int64_t per_wave = (int64_t)sm_count() * per_sm;
    const int64_t items = ((L + sru::kScanT - 1) / sru::kScanT) * ctas;
    const int64_t waves = (items + per_wave - 1) / per_wave;
    return waves * wave_chunks < (L + sru::kChunkT - 1) / sru::kChunkT;
}
int fwd_scan_resident(int u_t) {
    if (u_t == SRU_BF16)
        return scan_resident(reinterpret_cast<const void*>(sru::sru_fwd_scan_kernel<__nv_bfloat16>),
                             sru::FwdScanLayout<__nv_bfloat16>::SMEM);
    return scan_resident(reinterpret_cast<const void*>(sru::sru_fwd_scan_kernel<float>),
                         sru::FwdScanLayout<float>::SMEM);
}
// (the first direction's kernel with a U-typed dU stands for every variant)
int bwd_scan_resident(int u_t, bool v_zero) {
    if (u_t == SRU_BF16)
        return v_zero ? scan_resident(reinterpret_cast<const void*>(
                                          sru::sru_bwd_scan_kernel<__nv_bfloat16, __nv_bfloat16, false, 0, true>),
                                      sru::BwdScanLayout<__nv_bfloat16, false>::SMEM)
                      : scan_resident(reinterpret_cast<const void*>(
                                          sru::sru_bwd_scan_kernel<__nv_bfloat16, __nv_bfloat16, false, 0, false>),
                                      sru::BwdScanLayout<__nv_bfloat16, false>::SMEM);
    return v_zero ? scan_resident(reinterpret_cast<const void*>(sru::sru_bwd_scan_kernel<float, float, false, 0, true>),
                                  sru::BwdScanLayout<float, false>::SMEM)
                  : scan_resident(reinterpret_cast<const void*>(sru::sru_bwd_scan_kernel<float, float, false, 0, false>),
                                  sru::BwdScanLayout<float, false>::SMEM);
}
bool use_fwd_scan(unsigned flags, int64_t L, int64_t B, int64_t d, int n_dir, int u_t) {
    if (!(flags & SRU_FLAG_V_ZERO)) return false;
    if (flags & SRU_FLAG_FORCE_SCAN) return true;
    if (flags & SRU_FLAG_FORCE_SEQUENTIAL) return false;
    return scan_candidate(B, d, n_dir) &&
           scan_pays(L, seq_ctas(B, d, n_dir), fwd_scan_resident(u_t), kScanWaveChunksFwd);
}
bool use_bwd_scan(unsigned flags, int64_t L, int64_t B, int64_t d, int n_dir, int u_t) {
    if (flags & SRU_FLAG_FORCE_SCAN) return true;
    if (flags & SRU_FLAG_FORCE_SEQUENTIAL) return false;
    // one direction per backward launch
    return scan_candidate(B, d, 1) &&
           scan_pays(L, seq_ctas(B, d, 1), bwd_scan_resident(u_t, (flags & SRU_FLAG_V_ZERO) != 0),
                     kScanWaveChunksBwd);
}
// Whether a workspace for these sizes and flags carries the scan regions: a
// superset of the layers that take a scan (it depends on sizes and flags only,
// not on the U dtype).
bool ws_has_scan(unsigned flags, int64_t L, int64_t B, int64_t d, int n_dir) {
    (void)L;
    (void)n_dir;
    if (flags & (SRU_FLAG_FORCE_SCAN | SRU_FLAG_V_ZERO)) return true;
    if (flags & SRU_FLAG_FORCE_SEQUENTIAL) return false;
    return scan_candidate(B, d, 1);
}

sru_status check_layer_sizes(int64_t L, int64_t B, int64_t d) {
    if (L < 0 || B < 0 || d < 1) return SRU_ERR_INVALID;
    if (d % 8 != 0) return SRU_ERR_UNSUPPORTED;
    if (B > 65535 || L > (int64_t)1 << 30 || d > (int64_t)1 << 24) return SRU_ERR_UNSUPPORTED;
    if (L * B >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
    return SRU_OK;
}

inline unsigned blocks_for(size_t n, unsigned threads) { return (unsigned)((n + threads - 1) / threads); }

// ------------------------------------------------------------- GEMM launch
// The CTA-pair kernel: 256 x 256 output tiles over two SMs; a K-major B
// operand is staged as 128 rows per CTA.
constexpr uint32_t kGemmBRows = (uint32_t)sru::gemm::P_CN;

// tail_split (pair kernel, OUT == kOutF32 only): the output tiles of the last,
// partial round of CTA pairs are cut in two k-pieces that add onto regions
// zeroed here first (see sru::gemm::pair_next).
template <bool A_MN, bool B_MN, int OUT>
sru_status launch_tc_gemm(const CUtensorMap& ma, const CUtensorMap& mb, void* out, int64_t R, int64_t C,
                          int64_t Kr, cudaStream_t st, int splits = 1, int64_t ldo = -1, bool tail_split = false) {
    if (ldo < 0) ldo = C;
    {
        auto kern = sru::gemm::tc_gemm_pair_kernel<A_MN, B_MN, OUT>;
        SRU_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), sru::gemm::P_SMEM_BYTES));
        // the output as the epilogue's TMA store target: boxes of 32 rows x 128 bytes
        // (64 bf16 or 32 fp32 columns), swizzled like the staging buffers
        CUtensorMap mo;
        {
            const bool bf = OUT == sru::gemm::kOutBF16;
            const uint64_t dims[2] = {(uint64_t)C, (uint64_t)R};
            const uint64_t strides[1] = {(uint64_t)ldo * (bf ? 2 : 4)};
            const uint32_t box[2] = {(uint32_t)sru::gemm::EpiChunk<OUT>::kCols, 32};
            if (!make_map(&mo, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, dims,
                          strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return SRU_ERR_INVALID;
        }
        const int64_t n_tiles = (C + sru::gemm::P_BN - 1) / sru::gemm::P_BN;
        const int64_t tiles = ((R + sru::gemm::P_BM - 1) / sru::gemm::P_BM) * n_tiles;
        const int64_t units = tiles * splits;
        const int64_t pairs = units < sm_count() / 2 ? units : sm_count() / 2;
        int tail_s = 0;
        const int64_t kblocks = (Kr + sru::gemm::BK - 1) / sru::gemm::BK;
        // the pairs past the Rt long pieces take q short pieces each at most (see
        // sru::gemm::pair_next).  The tail is split for q <= 2 (a partial round of at
        // most two thirds of the pairs) with two k-blocks or more per piece.  q = 3
        // was measured without gain (M16384 N512 K6144: 78.2 us against 77.8 us
        // unsplit, before the zeroing's 6.3 us).
        const int64_t Rt = tiles % pairs;
        const int64_t q = Rt > 0 && Rt < pairs ? (Rt + (pairs - Rt) - 1) / (pairs - Rt) : 0;
        if (tail_split && OUT == sru::gemm::kOutF32 && splits == 1 && tiles > pairs && Rt != 0 && q <= 2 &&
            kblocks >= 2 * (q + 1)) {
            const int64_t F = tiles / pairs;
            tail_s = (int)(kblocks / (q + 1));
            const dim3 zgrid((unsigned)Rt, (unsigned)(sru::gemm::P_BM / sru::gemm::kZeroRows));
            sru::gemm::zero_tail_tiles_kernel<<<zgrid, 256, 0, st>>>(reinterpret_cast<float*>(out), (int)R, (int)C,
                                                                   (long long)ldo, (int)n_tiles, (int)(F * pairs));
            SRU_CUDA_TRY(cudaGetLastError());
        }
        kern<<<(unsigned)(2 * pairs), sru::gemm::THREADS, sru::gemm::P_SMEM_BYTES, st>>>(
            ma, mb, mo, (int)R, (int)C, (int)Kr, splits, 1, tail_s, 0);
    }
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

// `batches` products of one shape in one launch of the pair kernel (operand
// maps from map_kmajor_b / map_mnmajor_b with the batch at coordinate BPA /
// BPB); product z writes out + z * out_bstride elements, rows ldo apart, by
// TMA stores through a 3-D output map (batch coordinate 1 when the batch
// stride is below the row stride, else 2).
// CAUSAL (square causal attention products, see sru::gemm::pair_unit): 1 = only
// the output tiles on or below the diagonal, 2 = reduction cut at each row
// tile's diagonal, 3 = reduction started at each row tile's diagonal.
template <bool A_MN, bool B_MN, int OUT, int BPA, int BPB, int CAUSAL, int BPO>
sru_status launch_batched_bpo(const CUtensorMap& ma, const CUtensorMap& mb, void* out, int64_t R, int64_t C,
                              int64_t Kr, int64_t ldo, int64_t batches, int64_t out_bstride, cudaStream_t st) {
    auto kern = sru::gemm::tc_gemm_pair_kernel<A_MN, B_MN, OUT, BPA, BPB, CAUSAL, BPO>;
    SRU_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), sru::gemm::P_SMEM_BYTES));
    const int64_t mt = (R + sru::gemm::P_BM - 1) / sru::gemm::P_BM, nt = (C + sru::gemm::P_BN - 1) / sru::gemm::P_BN;
    if (CAUSAL == 1 && R != C) return SRU_ERR_UNSUPPORTED;
    const int64_t units = (CAUSAL == 1 ? mt * (mt + 1) / 2 : mt * nt) * batches;
    if (units >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
    const int64_t pairs = units < sm_count() / 2 ? units : sm_count() / 2;
    CUtensorMap mo;
    {
        const bool bf = OUT == sru::gemm::kOutBF16;
        const uint64_t es = bf ? 2 : 4;
        const uint32_t kc = (uint32_t)sru::gemm::EpiChunk<OUT>::kCols;
        uint64_t dims[3], strides[2];
        uint32_t box[3];
        if (BPO == 1) {
            dims[0] = (uint64_t)C; dims[1] = (uint64_t)batches; dims[2] = (uint64_t)R;
            strides[0] = (uint64_t)out_bstride * es; strides[1] = (uint64_t)ldo * es;
            box[0] = kc; box[1] = 1; box[2] = 32;
        } else {
            dims[0] = (uint64_t)C; dims[1] = (uint64_t)R; dims[2] = (uint64_t)batches;
            strides[0] = (uint64_t)ldo * es; strides[1] = (uint64_t)out_bstride * es;
            box[0] = kc; box[1] = 32; box[2] = 1;
        }
        if (!make_map(&mo, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, dims,
                      strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SRU_ERR_INVALID;
    }
    kern<<<(unsigned)(2 * pairs), sru::gemm::THREADS, sru::gemm::P_SMEM_BYTES, st>>>(
        ma, mb, mo, (int)R, (int)C, (int)Kr, 1, (int)batches, 0, 0);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

template <bool A_MN, bool B_MN, int OUT, int BPA, int BPB, int CAUSAL = 0>
sru_status launch_tc_gemm_batched(const CUtensorMap& ma, const CUtensorMap& mb, void* out, int64_t R, int64_t C,
                                  int64_t Kr, int64_t ldo, int64_t batches, int64_t out_bstride, cudaStream_t st) {
    if (out_bstride < ldo) {
        if (C > out_bstride) return SRU_ERR_INVALID;  // the batches' columns would overlap
        return launch_batched_bpo<A_MN, B_MN, OUT, BPA, BPB, CAUSAL, 1>(ma, mb, out, R, C, Kr, ldo, batches,
                                                                       out_bstride, st);
    }
    return launch_batched_bpo<A_MN, B_MN, OUT, BPA, BPB, CAUSAL, 2>(ma, mb, out, R, C, Kr, ldo, batches, out_bstride,
                                                                   st);
}

// Batched K-major operand: element (row r, k) of batch z at
// p[z * batch_ld + r * row_ld + k]; the batch is coordinate bpos (1: dims
// (K, batches, rows), 2: dims (K, rows, batches)) -- whichever keeps the
// strides increasing.
bool map_kmajor_b(CUtensorMap* m, const void* p, int64_t rows, int64_t K, int64_t row_ld, int64_t batches,
                  int64_t batch_ld, uint32_t box_rows, int bpos) {
    if (bpos == 1) {
        const uint64_t dims[3] = {(uint64_t)K, (uint64_t)batches, (uint64_t)rows};
        const uint64_t strides[2] = {(uint64_t)batch_ld * 2, (uint64_t)row_ld * 2};
        const uint32_t box[3] = {64, 1, box_rows};
        return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    const uint64_t dims[3] = {(uint64_t)K, (uint64_t)rows, (uint64_t)batches};
    const uint64_t strides[2] = {(uint64_t)row_ld * 2, (uint64_t)batch_ld * 2};
    const uint32_t box[3] = {64, box_rows, 1};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// Batched MN-major operand: element (r, k) of batch z at p[z * batch_ld + k * ld + r].
bool map_mnmajor_b(CUtensorMap* m, const void* p, int64_t rows, int64_t K, int64_t ld, int64_t batches,
                   int64_t batch_ld, int bpos) {
    if (bpos == 1) {
        const uint64_t dims[3] = {(uint64_t)rows, (uint64_t)batches, (uint64_t)K};
        const uint64_t strides[2] = {(uint64_t)batch_ld * 2, (uint64_t)ld * 2};
        const uint32_t box[3] = {64, 1, 64};
        return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    const uint64_t dims[3] = {(uint64_t)rows, (uint64_t)K, (uint64_t)batches};
    const uint64_t strides[2] = {(uint64_t)ld * 2, (uint64_t)batch_ld * 2};
    const uint32_t box[3] = {64, 64, 1};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// K-major operand (rows x K), contiguous K, rows ld elements apart (ld >= K;
// default K): box (64, box_rows)
bool map_kmajor(CUtensorMap* m, const void* p, int64_t rows, int64_t K, uint32_t box_rows, int64_t ld = -1) {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
    const uint64_t strides[1] = {(uint64_t)(ld < 0 ? K : ld) * 2};
    const uint32_t box[2] = {64, box_rows};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// MN-major operand: element (r, k) at p[k * ld + r], rows r contiguous: box (64, 64)
bool map_mnmajor(CUtensorMap* m, const void* p, int64_t rows, int64_t K, int64_t ld) {
    const uint64_t dims[2] = {(uint64_t)rows, (uint64_t)K};
    const uint64_t strides[1] = {(uint64_t)ld * 2};
    const uint32_t box[2] = {64, 64};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

sru_status launch_simt(const float* A, int64_t a_rs, int64_t a_ks, const float* Bm, int64_t b_rs, int64_t b_ks,
                       float* out, int64_t R, int64_t C, int64_t K, int accumulate, cudaStream_t st) {
    dim3 grid((unsigned)((C + sru::gemm::ST - 1) / sru::gemm::ST), (unsigned)((R + sru::gemm::ST - 1) / sru::gemm::ST));
    if (grid.y > 65535) return SRU_ERR_UNSUPPORTED;
    sru::gemm::simt_gemm_f32_kernel<<<grid, 256, 0, st>>>(A, a_rs, a_ks, Bm, b_rs, b_ks, out, C, (int)R, (int)C,
                                                          (int)K, accumulate);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

sru_status zero_f32(float* p, size_t n, cudaStream_t st) {
    if (n == 0) return SRU_OK;
    sru::sru_fill_f32_kernel<<<blocks_for(n, 256), 256, 0, st>>>(p, n, 0.f);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

// ------------------------------------------------------- recurrence launch
struct RecMaps {
    CUtensorMap u, x, dh;
    CUtensorMap du, dxo;  // backward outputs, for the kernels that store them with TMA
    CUtensorMap h;        // forward output, likewise
};

bool map_u_tensor(CUtensorMap* m, const void* U, int u_t, int64_t L, int64_t B, int64_t d, int n_dir, int cj) {
    const uint64_t es = u_t == SRU_BF16 ? 2 : 4;
    const uint64_t dims[4] = {(uint64_t)d, 3, (uint64_t)(B * n_dir), (uint64_t)L};
    const uint64_t strides[3] = {(uint64_t)d * es, (uint64_t)3 * d * es, (uint64_t)B * n_dir * 3 * d * es};
    const uint32_t box[4] = {(uint32_t)cj, 3, 1, (uint32_t)sru::kChunkT};
    return make_map(m, u_t == SRU_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, U,
                    dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}
// fp32 (L, rows, d) tensor with tiles (cj, 1, T)
bool map_f32_rows(CUtensorMap* m, const float* p, int64_t L, int64_t rows, int64_t d, int cj) {
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)rows, (uint64_t)L};
    const uint64_t strides[2] = {(uint64_t)d * 4, (uint64_t)rows * d * 4};
    const uint32_t box[3] = {(uint32_t)cj, 1, (uint32_t)sru::kChunkT};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// CTAs of a kernel (launched with `threads` threads and `smem` bytes of
// dynamic shared memory) that fit on one SM; cached per (kernel, device).
int resident_ctas(const void* kernel, int threads, size_t smem) {
    static std::mutex mu;
    static const void* known_kernel[256];
    static int known_dev[256], known_n[256];
    static int nknown = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < nknown; ++i)
            if (known_kernel[i] == kernel && known_dev[i] == dev) return known_n[i];
    }
    int n = 0;
    if (ensure_smem(kernel, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
        n = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (nknown < 256) {
        known_kernel[nknown] = kernel;
        known_dev[nknown] = dev;
        known_n[nknown] = n;
        ++nknown;
    }
    return n;
}

// Stage count for a sequential-kernel grid of `ctas` CTAs: the fewest waves
// of resident CTAs, then the deepest ring.  resident[S] = CTAs per SM at S
// stages (S = 2 .. smax).
int pick_stages(int64_t ctas, const int* resident, int smax) {
    int best = smax;
    int64_t best_waves = INT64_MAX;
    for (int S = smax; S >= 2; --S) {
        if (resident[S] <= 0) continue;
        const int64_t per_wave = (int64_t)sm_count() * resident[S];
        const int64_t waves = (ctas + per_wave - 1) / per_wave;
        if (waves < best_waves) {
            best_waves = waves;
            best = S;
        }
    }
    return best;
}

// Channels per CTA of the sequential kernels: 64 (one warp, two channels per
// thread).  Measured on B200, a 32-channel (half-warp) CTA was no faster where
// the 64-channel grid leaves SMs idle (L256 B32 d512: 38.9 us forward and
// 48.1 us backward at either width) and slower for the backward of dense grids
// (L1024 B16 d2048: 163 -> 194 us), so the kernels are built at 64 only.
constexpr int kSeqCJ = 64;
int seq_cj(int64_t, int64_t, int) { return kSeqCJ; }

template <typename UT, int CJ, int S, bool STAGE_H = false>
sru_status launch_fwd_seq_s(const RecMaps& mp, const float* v, const float* b, const float* c0, const uint8_t* mask,
                            float* h, float* c_T, float* ckpt, const int* order, int64_t L, int64_t B, int64_t d,
                            int n_dir, float alpha, cudaStream_t st) {
    using Lay = sru::FwdLayout<UT, CJ, S>;
    auto kern = sru::sru_fwd_seq_kernel<UT, CJ, S, STAGE_H>;
    SRU_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), Lay::SMEM));
    const dim3 grid = order != nullptr ? dim3((unsigned)((d + CJ - 1) / CJ), (unsigned)(B * n_dir), 1)
                                       : dim3((unsigned)((d + CJ - 1) / CJ), (unsigned)B, (unsigned)n_dir);
    kern<<<grid, CJ / 2, Lay::SMEM, st>>>(mp.u, mp.x, mp.h, v, b, c0, mask, h, c_T, ckpt, order, (int)L, (int)B,
                                              (int)d, n_dir, alpha);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

template <typename UT, int CJ, int S>
int fwd_resident() {
    return resident_ctas(reinterpret_cast<const void*>(sru::sru_fwd_seq_kernel<UT, CJ, S>), CJ / 2,
                         sru::FwdLayout<UT, CJ, S>::SMEM);
}

// A padded layer whose grid needs more than one wave of resident CTAs takes
// its (batch row, direction) streams longest first (sru_length_order_kernel,
// into the workspace's order region); returns the order, or null to keep the
// natural one.
sru_status maybe_order(const uint8_t* mask, int* order_ws, int64_t L, int64_t B, int n_dir, int64_t ctas,
                       int64_t per_wave, cudaStream_t st, const int** order) {
    *order = nullptr;
    if (mask == nullptr || order_ws == nullptr || B > sru::kOrderMaxB || B < 2 || ctas <= per_wave) return SRU_OK;
    sru::sru_length_order_kernel<<<1, sru::kOrderThreads, 0, st>>>(mask, (int)L, (int)B, n_dir, order_ws);
    SRU_CUDA_TRY(cudaGetLastError());
    *order = order_ws;
    return SRU_OK;
}

template <typename UT, int CJ>
sru_status launch_fwd_seq(const RecMaps& mp, const float* v, const float* b, const float* c0, const uint8_t* mask,
                          float* h, float* c_T, float* ckpt, int* order_ws, int64_t L, int64_t B, int64_t d, int n_dir,
                          float alpha, cudaStream_t st) {
    static_assert(sru::kFwdStages == 4, "stage dispatch below covers 2..4");
    const int resident[5] = {0, 0, fwd_resident<UT, CJ, 2>(), fwd_resident<UT, CJ, 3>(), fwd_resident<UT, CJ, 4>()};
    const int64_t ctas = ((d + CJ - 1) / CJ) * B * n_dir;
    const int S = pick_stages(ctas, resident, 4);
    const int* order = nullptr;
    sru_status s = maybe_order(mask, order_ws, L, B, n_dir, ctas, (int64_t)sm_count() * resident[S], st, &order);
    if (s != SRU_OK) return s;
    // h through TMA stores: for unmasked grids of about 5 or more CTAs per SM (measured)
    if (S >= 3 && mask == nullptr && ctas * 10 >= (int64_t)sm_count() * 48)
        return S == 3 ? launch_fwd_seq_s<UT, CJ, 3, true>(mp, v, b, c0, mask, h, c_T, ckpt, order, L, B, d, n_dir, alpha, st)
                      : launch_fwd_seq_s<UT, CJ, 4, true>(mp, v, b, c0, mask, h, c_T, ckpt, order, L, B, d, n_dir, alpha, st);
    switch (S) {
        case 2: return launch_fwd_seq_s<UT, CJ, 2>(mp, v, b, c0, mask, h, c_T, ckpt, order, L, B, d, n_dir, alpha, st);
        case 3: return launch_fwd_seq_s<UT, CJ, 3>(mp, v, b, c0, mask, h, c_T, ckpt, order, L, B, d, n_dir, alpha, st);
        default: return launch_fwd_seq_s<UT, CJ, 4>(mp, v, b, c0, mask, h, c_T, ckpt, order, L, B, d, n_dir, alpha, st);
    }
}

template <typename UT, typename DUT, bool ACC, int DIR, int CJ, int S>
sru_status launch_bwd_seq_s(const RecMaps& mp, const float* v, const float* b, const uint8_t* mask,
                            const float* ckpt, const float* dc_T, DUT* dU, float* dx, double* partial, float* dc0,
                            const int* order, int64_t L, int64_t B, int64_t d, int n_dir, float alpha, cudaStream_t st) {
    using Lay = sru::BwdLayout<UT, ACC, CJ, S>;
    auto kern = sru::sru_bwd_seq_kernel<UT, DUT, ACC, DIR, CJ, S>;
    SRU_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), Lay::SMEM));
    dim3 grid((unsigned)((d + CJ - 1) / CJ), (unsigned)B, 1);
    kern<<<grid, CJ / 2, Lay::SMEM, st>>>(mp.u, mp.x, mp.dh, mp.du, mp.dxo, v, b, mask, ckpt, dc_T, dU, dx, partial, dc0,
                                              order, (int)L, (int)B, (int)d, n_dir, alpha);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

template <typename UT, typename DUT, bool ACC, int DIR, int CJ, int S>
int bwd_resident() {
    return resident_ctas(reinterpret_cast<const void*>(sru::sru_bwd_seq_kernel<UT, DUT, ACC, DIR, CJ, S>),
                         CJ / 2, sru::BwdLayout<UT, ACC, CJ, S>::SMEM);
}

// One direction's backward launch.  ACC: dx += this direction's part.
template <typename UT, typename DUT, bool ACC, int DIR, int CJ>
sru_status launch_bwd_seq_dir(const RecMaps& mp, const float* v, const float* b, const uint8_t* mask,
                              const float* ckpt, const float* dc_T, DUT* du, float* dx, double* partial, float* dc0,
                              int* order_ws, const int** order, int64_t L, int64_t B, int64_t d, int n_dir, float alpha,
                              cudaStream_t st) {
    static_assert(sru::kBwdStages == 3, "stage dispatch below covers 2..3");
    const int resident[4] = {0, 0, bwd_resident<UT, DUT, ACC, DIR, CJ, 2>(), bwd_resident<UT, DUT, ACC, DIR, CJ, 3>()};
    const int64_t ctas = ((d + CJ - 1) / CJ) * B;
    const int S = pick_stages(ctas, resident, 3);
    if (DIR == 0) {  // one order for both directions' launches
        sru_status s = maybe_order(mask, order_ws, L, B, n_dir, ctas, (int64_t)sm_count() * resident[S], st, order);
        if (s != SRU_OK) return s;
    }
    if (S == 2)
        return launch_bwd_seq_s<UT, DUT, ACC, DIR, CJ, 2>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, *order, L, B,
                                                      d, n_dir, alpha, st);
    return launch_bwd_seq_s<UT, DUT, ACC, DIR, CJ, 3>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, *order, L, B, d,
                                                  n_dir, alpha, st);
}

template <typename UT, typename DUT, int CJ>
sru_status launch_bwd_seq(const RecMaps& mp, const float* v, const float* b, const uint8_t* mask, const float* ckpt,
                          const float* dc_T, void* dU, float* dx, double* partial, float* dc0, int* order_ws,
                          int64_t L, int64_t B, int64_t d, int n_dir, float alpha, cudaStream_t st) {
    DUT* du = reinterpret_cast<DUT*>(dU);
    const int* order = nullptr;
    sru_status s = launch_bwd_seq_dir<UT, DUT, false, 0, CJ>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, order_ws,
                                                         &order, L, B, d, n_dir, alpha, st);
    if (s != SRU_OK || n_dir == 1) return s;
    return launch_bwd_seq_dir<UT, DUT, true, 1, CJ>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, order_ws, &order, L,
                                                B, d, n_dir, alpha, st);
}

sru_status reset_scan_flags(unsigned* flags, int64_t n, cudaStream_t st) {
    sru::sru_scan_reset_kernel<<<blocks_for((size_t)n, 256), 256, 0, st>>>(flags, (int)n);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

template <typename UT>
sru_status launch_fwd_scan(const RecMaps& mp, const float* b, const float* c0, const uint8_t* mask, float* h,
                           float* c_T, float* ckpt, const sru::ScanState& ss, int64_t L, int64_t B, int64_t d,
                           int n_dir, float alpha, cudaStream_t st) {
    using Lay = sru::FwdScanLayout<UT>;
    auto kern = sru::sru_fwd_scan_kernel<UT>;
    SRU_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), Lay::SMEM));
    const int64_t items = scan_chunks(L) * ((d + sru::kRecCJ - 1) / sru::kRecCJ) * B * n_dir;
    if (items >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
    sru_status s = reset_scan_flags(ss.flags, items + 1, st);
    if (s != SRU_OK) return s;
    kern<<<(unsigned)items, sru::kScanThreads, Lay::SMEM, st>>>(mp.u, mp.x, b, c0, mask, h, c_T, ckpt, ss, (int)L,
                                                           (int)B, (int)d, n_dir, alpha);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

template <typename UT, typename DUT, bool ACC, int DIR, bool VZ>
sru_status launch_bwd_scan_dir(const RecMaps& mp, const float* v, const float* b, const uint8_t* mask,
                               const float* ckpt,
                               const float* dc_T, DUT* dU, float* dx, double* partial, float* dc0,
                               const sru::ScanState& ss, int64_t L, int64_t B, int64_t d, int n_dir, float alpha,
                               cudaStream_t st) {
    using Lay = sru::BwdScanLayout<UT, ACC>;
    auto kern = sru::sru_bwd_scan_kernel<UT, DUT, ACC, DIR, VZ>;
    SRU_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), Lay::SMEM));
    const int64_t items = scan_chunks(L) * ((d + sru::kRecCJ - 1) / sru::kRecCJ) * B;
    if (items >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
    sru_status s = reset_scan_flags(ss.flags, items + 1, st);
    if (s != SRU_OK) return s;
    kern<<<(unsigned)items, sru::kScanThreads, Lay::SMEM, st>>>(mp.u, mp.x, mp.dh, v, b, mask, ckpt, dc_T, dU, dx,
                                                           partial, dc0, ss, (int)L, (int)B, (int)d, n_dir, alpha);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

template <typename UT, typename DUT, bool VZ>
sru_status launch_bwd_scan_vz(const RecMaps& mp, const float* v, const float* b, const uint8_t* mask,
                              const float* ckpt, const float* dc_T, DUT* du, float* dx, double* partial, float* dc0,
                              const sru::ScanState& ss, int64_t L, int64_t B, int64_t d, int n_dir, float alpha,
                              cudaStream_t st) {
    sru_status s = launch_bwd_scan_dir<UT, DUT, false, 0, VZ>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, ss,
                                                             L, B, d, n_dir, alpha, st);
    if (s != SRU_OK || n_dir == 1) return s;
    return launch_bwd_scan_dir<UT, DUT, true, 1, VZ>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, ss, L, B, d,
                                                    n_dir, alpha, st);
}

// v_zero: the caller asserted v == 0 (SRU_FLAG_V_ZERO), so the chunk maps need no state.
template <typename UT, typename DUT>
sru_status launch_bwd_scan(const RecMaps& mp, const float* v, const float* b, const uint8_t* mask, const float* ckpt,
                           const float* dc_T, void* dU, float* dx, double* partial, float* dc0,
                           const sru::ScanState& ss, int64_t L, int64_t B, int64_t d, int n_dir, float alpha,
                           cudaStream_t st, bool v_zero) {
    DUT* du = reinterpret_cast<DUT*>(dU);
    if (v_zero)
        return launch_bwd_scan_vz<UT, DUT, true>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, ss, L, B, d,
                                                 n_dir, alpha, st);
    return launch_bwd_scan_vz<UT, DUT, false>(mp, v, b, mask, ckpt, dc_T, du, dx, partial, dc0, ss, L, B, d, n_dir,
                                              alpha, st);
}

// ------------------------------------------------------------ decode step
template <int NB>
sru_status launch_decode_nb(const void* X_t, const void* W, const float* x_t, const float* v, const float* b,
                            float* c, float* h_t, int64_t B, int64_t d, float alpha, cudaStream_t st) {
    const dim3 grid((unsigned)((d + sru::kDecWarps - 1) / sru::kDecWarps), (unsigned)((B + NB - 1) / NB));
    sru::sru_decode_step_kernel<NB><<<grid, sru::kDecThreads, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(X_t), reinterpret_cast<const __nv_bfloat16*>(W), x_t, v, b, c, h_t,
        (int)B, (int)d, alpha);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

// Batch rows per pass over W: the smallest instantiated count covering B (at most 16).
int decode_rows_per_pass(int64_t B) {
    int nb = 1;
    while (nb < B && nb < sru::kDecMaxNB) nb *= 2;
    return nb;
}

}  // namespace

// ---------------------------------------------------------------------------
// Static scratch of the allocation-free entry point sru_forward_scan_noalloc.
// Every GPU that loads this library holds these 8 MiB until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Scan flags, ticket and aggregates of `items` work items carved from the scratch.
size_t noalloc_scan_bytes(int64_t items, size_t* agg_a_off, size_t* agg_b_off, size_t* prefix_off) {
    size_t off = round256((size_t)(items + 1) * sizeof(unsigned));
    *agg_a_off = off;
    off += round256((size_t)items * sru::kRecCJ * sizeof(float));
    *agg_b_off = off;
    off += round256((size_t)items * sru::kRecCJ * sizeof(float));
    *prefix_off = off;
    off += round256((size_t)items * sru::kRecCJ * sizeof(float));
    return off;
}

// Device address of the scratch on the current device, looked up once per
// device.  In host code g_noalloc_scratch names a host-side stand-in, never
// the device array, so kernels only ever receive this looked-up address.  The
// lookup is not a stream operation, but it may load the library's module on
// the device, which a stream capture in progress does not allow: a first call
// on a device made while `st` is capturing is refused with SRU_ERR_INVALID.
sru_status noalloc_scratch_address(cudaStream_t st, void** out) {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice);
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        e = cudaStreamIsCapturing(st, &cs);
        if (e != cudaSuccess) return cuda_fail(e);
        if (cs != cudaStreamCaptureStatusNone) return SRU_ERR_INVALID;  // first call during a capture
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        addr[dev] = p;
    }
    *out = addr[dev];
    return SRU_OK;
}

// CTA pairs of the fused forward that the device can hold at once (the
// kernel hands the state between CTAs, so its whole grid must be resident):
// the occupancy calculator's count of co-resident 2-CTA clusters, cached per
// device.
int64_t fused_resident_pairs() {
    static std::mutex mu;
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        const void* kern = reinterpret_cast<const void*>(sru::fused::sru_fused_fwd_kernel);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * (sm_count() / 2)), 1, 1);
        cfg.blockDim = dim3(sru::fused::kThreads, 1, 1);
        cfg.dynamicSmemBytes = sru::fused::kSmemBytes;
        int n = 0;
        if (ensure_smem(kern, sru::fused::kSmemBytes) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess)
            n = 0;
        cache[dev] = n > 0 ? (n < sm_count() / 2 ? n : sm_count() / 2) : -1;
    }
    return cache[dev];
}

}  // namespace

// =========================================================================
// grid: two CTAs per SM (one for the widest rows), at most one per kNormRows
// rows (the slices the workspace holds); returns the slices written
template <int NV>
unsigned norm_backward_params_reg(const float* dR, const __nv_bfloat16* Q, const float* A, float alpha, const float* g,
                                  float* dQ, __nv_bfloat16* dA, float2* stats, float* part, int64_t M, int64_t dp,
                                  cudaStream_t st) {
    const unsigned per_sm = NV <= 4 ? 2u : 1u;
    unsigned grid = (unsigned)sm_count() * per_sm;
    const unsigned cap = blocks_for((size_t)M, sru::kNormRows);
    if (grid > cap) grid = cap;
    sru::sru_norm_backward_params_reg_kernel<NV><<<grid, sru::kRowWarps * 32, 0, st>>>(dR, Q, A, alpha, g, dQ, dA,
                                                                                     stats, part, (int)M, (int)dp);
    return grid;
}
template <int NV>
void norm_backward_reg(const float* dR, const __nv_bfloat16* Q, const float* A, float alpha, const float* g, float* dQ,
                       __nv_bfloat16* dA, float2* stats, int64_t M, int64_t dp, cudaStream_t st) {
    sru::sru_norm_backward_reg_kernel<NV><<<blocks_for((size_t)M, sru::kRowWarps), sru::kRowWarps * 32, 0, st>>>(
        dR, Q, A, alpha, g, dQ, dA, stats, (int)M, (int)dp);
}
sru_status launch_norm_backward(const float* dR, const __nv_bfloat16* Q, const float* A, float alpha, const float* g,
                                float* dQ, __nv_bfloat16* dA, float2* stats, int64_t M, int64_t dp, cudaStream_t st) {
    const int64_t nv = (dp + 127) / 128;
    if (nv <= 1) norm_backward_reg<1>(dR, Q, A, alpha, g, dQ, dA, stats, M, dp, st);
    else if (nv <= 2) norm_backward_reg<2>(dR, Q, A, alpha, g, dQ, dA, stats, M, dp, st);
    else if (nv <= 4) norm_backward_reg<4>(dR, Q, A, alpha, g, dQ, dA, stats, M, dp, st);
    else if (nv <= 8) norm_backward_reg<8>(dR, Q, A, alpha, g, dQ, dA, stats, M, dp, st);
    else
        sru::sru_norm_backward_kernel<<<blocks_for((size_t)M, sru::kRowWarps), sru::kRowWarps * 32, 0, st>>>(
            dR, Q, A, alpha, g, dQ, dA, stats, (int)M, (int)dp);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}
// The row-wise steps: the register-resident kernels for rows that fit (scores
// rows of L <= 2048, d' <= 1024), the streaming ones otherwise.
template <int NV>
void softmax_reg(const float* S, __nv_bfloat16* P, int64_t L, int64_t rows, float scale, int causal, cudaStream_t st) {
    sru::sru_softmax_rows_reg_kernel<NV><<<blocks_for((size_t)rows, sru::kRowWarps), sru::kRowWarps * 32, 0, st>>>(
        S, P, (int)L, (int)rows, scale, causal);
}
sru_status launch_softmax_rows(const float* S, __nv_bfloat16* P, int64_t L, int64_t rows, float scale, int causal,
                               cudaStream_t st) {
    const int64_t nv = (L + 127) / 128;
    if (nv <= 1) softmax_reg<1>(S, P, L, rows, scale, causal, st);
    else if (nv <= 2) softmax_reg<2>(S, P, L, rows, scale, causal, st);
    else if (nv <= 4) softmax_reg<4>(S, P, L, rows, scale, causal, st);
    else if (nv <= 8) softmax_reg<8>(S, P, L, rows, scale, causal, st);
    else if (nv <= 16) softmax_reg<16>(S, P, L, rows, scale, causal, st);
    else
        sru::sru_softmax_rows_kernel<<<blocks_for((size_t)rows, sru::kRowWarps), sru::kRowWarps * 32, 0, st>>>(
            S, P, (int)L, (int)rows, scale, causal);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}
template <int NV>
void softmax_backward_reg(const float* dP, const __nv_bfloat16* P, __nv_bfloat16* dS, int64_t L, int64_t rows,
                          float scale, int causal, cudaStream_t st) {
    sru::sru_softmax_backward_rows_reg_kernel<NV>
        <<<blocks_for((size_t)rows, sru::kRowWarps), sru::kRowWarps * 32, 0, st>>>(dP, P, dS, (int)L, (int)rows,
                                                                                  scale, causal);
}
sru_status launch_softmax_backward_rows(const float* dP, const __nv_bfloat16* P, __nv_bfloat16* dS, int64_t L,
                                        int64_t rows, float scale, int causal, cudaStream_t st) {
    const int64_t nv = (L + 127) / 128;
    if (nv <= 1) softmax_backward_reg<1>(dP, P, dS, L, rows, scale, causal, st);
    else if (nv <= 2) softmax_backward_reg<2>(dP, P, dS, L, rows, scale, causal, st);
    else if (nv <= 4) softmax_backward_reg<4>(dP, P, dS, L, rows, scale, causal, st);
    else if (nv <= 8) softmax_backward_reg<8>(dP, P, dS, L, rows, scale, causal, st);
    else if (nv <= 16) softmax_backward_reg<16>(dP, P, dS, L, rows, scale, causal, st);
    else
        sru::sru_softmax_backward_rows_kernel<<<blocks_for((size_t)rows, sru::kRowWarps), sru::kRowWarps * 32, 0,
                                                st>>>(dP, P, dS, (int)L, (int)rows, scale, causal);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}
template <int NV>
void residual_norm_reg(const __nv_bfloat16* Q, const float* A, float alpha, const float* g, const float* b,
                       __nv_bfloat16* R, int64_t M, int64_t dp, cudaStream_t st) {
    sru::sru_residual_norm_reg_kernel<NV><<<blocks_for((size_t)M, sru::kRowWarps), sru::kRowWarps * 32, 0, st>>>(
        Q, A, alpha, g, b, R, (int)M, (int)dp);
}
sru_status launch_residual_norm(const __nv_bfloat16* Q, const float* A, float alpha, const float* g, const float* b,
                                __nv_bfloat16* R, int64_t M, int64_t dp, cudaStream_t st) {
    const int64_t nv = (dp + 127) / 128;
    if (nv <= 1) residual_norm_reg<1>(Q, A, alpha, g, b, R, M, dp, st);
    else if (nv <= 2) residual_norm_reg<2>(Q, A, alpha, g, b, R, M, dp, st);
    else if (nv <= 4) residual_norm_reg<4>(Q, A, alpha, g, b, R, M, dp, st);
    else if (nv <= 8) residual_norm_reg<8>(Q, A, alpha, g, b, R, M, dp, st);
    else
        sru::sru_residual_norm_kernel<<<blocks_for((size_t)M, sru::kRowWarps), sru::kRowWarps * 32, 0, st>>>(
            Q, A, alpha, g, b, R, (int)M, (int)dp);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

extern "C" {

const char* sru_status_string(int status) {
    switch (status) {
        case SRU_OK: return "SRU_OK";
        case SRU_ERR_INVALID: return "SRU_ERR_INVALID: bad pointer, size, alignment or dtype";
        case SRU_ERR_CUDA: return "SRU_ERR_CUDA: a CUDA call failed";
        case SRU_ERR_TIMEOUT: return "SRU_ERR_TIMEOUT: a bounded device-side wait expired";
        case SRU_ERR_UNSUPPORTED: return "SRU_ERR_UNSUPPORTED: request outside the library's limits";
        default: return "unknown sru_status";
    }
}

int sru_get_last_cuda_error(void) { return g_last_cuda_error; }

int sru_version(void) { return 100; }

size_t sru_workspace_bytes(int64_t L, int64_t B, int64_t d, int bidirectional, unsigned flags) {
    if (check_layer_sizes(L, B, d) != SRU_OK) return 0;
    return ws_layout(L, B, d, bidirectional ? 2 : 1, flags).total;
}

sru_status sru_project(const void* X, int x_t, const void* W, int w_t, void* U, int u_t, int64_t M, int64_t N,
                       int64_t K, void* stream) {
    if (M < 0 || N < 0 || K < 0) return SRU_ERR_INVALID;
    if (M == 0 || N == 0) return SRU_OK;
    if (!X || !W || !U || !aligned16(X) || !aligned16(W) || !aligned16(U)) return SRU_ERR_INVALID;
    if (K % 8 != 0 || N % 8 != 0) return SRU_ERR_UNSUPPORTED;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    if (x_t == SRU_F32 && w_t == SRU_F32 && u_t == SRU_F32) {
        if (K == 0) return zero_f32(reinterpret_cast<float*>(U), (size_t)M * N, st);
        return launch_simt(reinterpret_cast<const float*>(X), K, 1, reinterpret_cast<const float*>(W), K, 1,
                           reinterpret_cast<float*>(U), M, N, K, 0, st);
    }
    if (x_t != SRU_BF16 || w_t != SRU_BF16 || (u_t != SRU_BF16 && u_t != SRU_F32)) return SRU_ERR_INVALID;
    if (K == 0) return SRU_ERR_UNSUPPORTED;
    CUtensorMap ma, mb;
    if (!map_kmajor(&ma, X, M, K, sru::gemm::P_CM) || !map_kmajor(&mb, W, N, K, kGemmBRows)) return SRU_ERR_INVALID;
    if (u_t == SRU_BF16) return launch_tc_gemm<false, false, sru::gemm::kOutBF16>(ma, mb, U, M, N, K, st);
    return launch_tc_gemm<false, false, sru::gemm::kOutF32>(ma, mb, U, M, N, K, st);
}

sru_status sru_project_backward(const void* dU, const void* X, const void* W, int t, float* dX, int accumulate,
                                float* dW, int64_t M, int64_t N, int64_t K, void* stream) {
    if (M < 0 || N < 0 || K < 0) return SRU_ERR_INVALID;
    if (!dU || !aligned16(dU)) return SRU_ERR_INVALID;
    if (dX && (!W || !aligned16(W) || !aligned16(dX))) return SRU_ERR_INVALID;
    if (dW && (!X || !aligned16(X) || !aligned16(dW))) return SRU_ERR_INVALID;
    if (K % 8 != 0 || N % 8 != 0) return SRU_ERR_UNSUPPORTED;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
    if (t != SRU_F32 && t != SRU_BF16) return SRU_ERR_INVALID;
    cudaStream_t st = as_stream(stream);
    if (K == 0) return SRU_OK;
    if (t == SRU_F32) {
        const float* du = reinterpret_cast<const float*>(dU);
        if (dX) {
            if (N == 0) {
                if (!accumulate) { sru_status s = zero_f32(dX, (size_t)M * K, st); if (s) return s; }
            } else if (M > 0) {
                sru_status s = launch_simt(du, N, 1, reinterpret_cast<const float*>(W), 1, K, dX, M, K, N, accumulate, st);
                if (s != SRU_OK) return s;
            }
        }
        if (dW && N > 0) {
            if (M == 0) return zero_f32(dW, (size_t)N * K, st);
            return launch_simt(du, 1, N, reinterpret_cast<const float*>(X), 1, K, dW, N, K, M, 0, st);
        }
        return SRU_OK;
    }
    // bf16 on the tensor cores
    if (dX && M > 0) {
        if (N == 0) {
            if (!accumulate) { sru_status s = zero_f32(dX, (size_t)M * K, st); if (s) return s; }
        } else {
            CUtensorMap ma, mb;
            // A = dU (M x N) K-major; B(c = k, red = n) = W[n][k]: MN-major with ld = K
            if (!map_kmajor(&ma, dU, M, N, sru::gemm::P_CM) || !map_mnmajor(&mb, W, K, N, K)) return SRU_ERR_INVALID;
            // written (not accumulated): the tiles of a last, partial round of CTA pairs are
            // cut in two k-pieces, as for dW
            sru_status s = accumulate ? launch_tc_gemm<false, true, sru::gemm::kOutF32Acc>(ma, mb, dX, M, K, N, st)
                                      : launch_tc_gemm<false, true, sru::gemm::kOutF32>(ma, mb, dX, M, K, N, st, 1,
                                                                                        -1, /*tail_split=*/true);
            if (s != SRU_OK) return s;
        }
    }
    if (dW && N > 0) {
        if (M == 0) return zero_f32(dW, (size_t)N * K, st);
        CUtensorMap ma, mb;
        // A(r = n, red = m) = dU[m][n]: MN-major, ld = N; B(c = k, red = m) = X[m][k]: MN-major, ld = K
        if (!map_mnmajor(&ma, dU, N, M, N) || !map_mnmajor(&mb, X, K, M, K)) return SRU_ERR_INVALID;
        return launch_tc_gemm<true, true, sru::gemm::kOutF32>(ma, mb, dW, N, K, M, st, 1, -1, /*tail_split=*/true);
    }
    return SRU_OK;
}

sru_status sru_forward(const void* U, int u_t, const float* x, const float* v, const float* b, const float* c0,
                       const uint8_t* mask, int64_t L, int64_t B, int64_t d, float alpha, int bidirectional,
                       unsigned flags, float* h, float* c_T, void* workspace, size_t workspace_bytes,
                       void* stream) {
    sru_status s = check_layer_sizes(L, B, d);
    if (s != SRU_OK) return s;
    if (u_t != SRU_F32 && u_t != SRU_BF16) return SRU_ERR_INVALID;
    const int n_dir = bidirectional ? 2 : 1;
    if (B == 0) return SRU_OK;
    if (!v || !b || !c_T) return SRU_ERR_INVALID;
    if (!aligned8_or_null(v) || !aligned8_or_null(b) || !aligned8_or_null(c0) || !aligned8_or_null(c_T))
        return SRU_ERR_INVALID;
    cudaStream_t st = as_stream(stream);
    if (L == 0) {
        const size_t n = (size_t)B * n_dir * d;
        sru::sru_copy_state_kernel<<<blocks_for(n, 256), 256, 0, st>>>(c0, c_T, n);
        SRU_CUDA_TRY(cudaGetLastError());
        return SRU_OK;
    }
    if (!U || !x || !h || !aligned16(U) || !aligned16(x) || !aligned16(h)) return SRU_ERR_INVALID;
    const WsLayout w = ws_layout(L, B, d, n_dir, flags);
    const bool scan = use_fwd_scan(flags, L, B, d, n_dir, u_t);
    if (workspace) {
        if (!aligned16(workspace) || workspace_bytes < w.total) return SRU_ERR_INVALID;
    } else if (scan) {
        return SRU_ERR_INVALID;  // the scan needs its flags and aggregates
    }
    const int cj = scan ? sru::kRecCJ : seq_cj(B, d, n_dir);  // TMA box width of the kernel that runs
    RecMaps mp;
    if (!map_u_tensor(&mp.u, U, u_t, L, B, d, n_dir, cj) || !map_f32_rows(&mp.x, x, L, B, d, cj) ||
        !map_f32_rows(&mp.h, h, L, B * n_dir, d, cj))
        return SRU_ERR_INVALID;
    float* ckpt = workspace ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.ckpt_off) : nullptr;
    int* order_ws = workspace ? reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + w.order_off) : nullptr;
    if (scan) {
        const sru::ScanState ss = scan_state(workspace, w, flags);
        if (u_t == SRU_BF16)
            return launch_fwd_scan<__nv_bfloat16>(mp, b, c0, mask, h, c_T, ckpt, ss, L, B, d, n_dir, alpha, st);
        return launch_fwd_scan<float>(mp, b, c0, mask, h, c_T, ckpt, ss, L, B, d, n_dir, alpha, st);
    }
    return u_t == SRU_BF16
               ? launch_fwd_seq<__nv_bfloat16, kSeqCJ>(mp, v, b, c0, mask, h, c_T, ckpt, order_ws, L, B, d, n_dir, alpha,
                                                        st)
               : launch_fwd_seq<float, kSeqCJ>(mp, v, b, c0, mask, h, c_T, ckpt, order_ws, L, B, d, n_dir, alpha, st);
}

sru_status sru_backward(const void* U, int u_t, const float* x, const float* v, const float* b, const float* c0,
                        const uint8_t* mask, int64_t L, int64_t B, int64_t d, float alpha, int bidirectional,
                        unsigned flags, const float* dh, const float* dc_T, void* workspace,
                        size_t workspace_bytes, void* dU, int du_t, float* dx, float* dv, float* db, float* dc0,
                        void* stream) {
    (void)c0;  // the forward's checkpoints already hold the state derived from c0
    sru_status s = check_layer_sizes(L, B, d);
    if (s != SRU_OK) return s;
    if (u_t != SRU_F32 && u_t != SRU_BF16) return SRU_ERR_INVALID;
    if (du_t != SRU_F32 && du_t != SRU_BF16) return SRU_ERR_INVALID;
    const int n_dir = bidirectional ? 2 : 1;
    if (!v || !b || !dv || !db) return SRU_ERR_INVALID;
    if (!aligned8_or_null(v) || !aligned8_or_null(b) || !aligned8_or_null(dc_T) || !aligned8_or_null(dv) ||
        !aligned8_or_null(db) || !aligned8_or_null(dc0))
        return SRU_ERR_INVALID;
    cudaStream_t st = as_stream(stream);
    if (B == 0 || L == 0) {
        // no steps: dv = db = 0, dc0 = dc_T
        s = zero_f32(dv, (size_t)n_dir * 2 * d, st);
        if (s == SRU_OK) s = zero_f32(db, (size_t)n_dir * 2 * d, st);
        if (s == SRU_OK && B > 0) {
            if (!dc0) return SRU_ERR_INVALID;
            const size_t n = (size_t)B * n_dir * d;
            sru::sru_copy_state_kernel<<<blocks_for(n, 256), 256, 0, st>>>(dc_T, dc0, n);
            SRU_CUDA_TRY(cudaGetLastError());
        }
        return s;
    }
    if (!U || !x || !dh || !workspace || !dU || !dx || !dc0) return SRU_ERR_INVALID;
    if (!aligned16(U) || !aligned16(x) || !aligned16(dh) || !aligned16(workspace) || !aligned16(dU) || !aligned16(dx))
        return SRU_ERR_INVALID;
    const WsLayout w = ws_layout(L, B, d, n_dir, flags);
    if (workspace_bytes < w.total) return SRU_ERR_INVALID;
    const bool scan = use_bwd_scan(flags, L, B, d, n_dir, u_t);
    const int cj = scan ? sru::kRecCJ : seq_cj(B, d, 1);
    RecMaps mp;
    if (!map_u_tensor(&mp.u, U, u_t, L, B, d, n_dir, cj) || !map_f32_rows(&mp.x, x, L, B, d, cj) ||
        !map_f32_rows(&mp.dh, dh, L, B * n_dir, d, cj) || !map_u_tensor(&mp.du, dU, du_t, L, B, d, n_dir, cj) ||
        !map_f32_rows(&mp.dxo, dx, L, B, d, cj))
        return SRU_ERR_INVALID;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const float* ckpt = reinterpret_cast<const float*>(ws + w.ckpt_off);
    double* partial = reinterpret_cast<double*>(ws + w.partial_off);
    int* order_ws = reinterpret_cast<int*>(ws + w.order_off);
    const bool ub = u_t == SRU_BF16, db16 = du_t == SRU_BF16;
    if (scan) {
        const sru::ScanState ss = scan_state(workspace, w, flags);
        if (ub)
            s = db16 ? launch_bwd_scan<__nv_bfloat16, __nv_bfloat16>(mp, v, b, mask, ckpt, dc_T, dU, dx, partial, dc0, ss,
                                                                     L, B, d, n_dir, alpha, st, (flags & SRU_FLAG_V_ZERO) != 0)
                     : launch_bwd_scan<__nv_bfloat16, float>(mp, v, b, mask, ckpt, dc_T, dU, dx, partial, dc0, ss, L, B,
                                                             d, n_dir, alpha, st, (flags & SRU_FLAG_V_ZERO) != 0);
        else
            s = db16 ? launch_bwd_scan<float, __nv_bfloat16>(mp, v, b, mask, ckpt, dc_T, dU, dx, partial, dc0, ss, L, B,
                                                             d, n_dir, alpha, st, (flags & SRU_FLAG_V_ZERO) != 0)
                     : launch_bwd_scan<float, float>(mp, v, b, mask, ckpt, dc_T, dU, dx, partial, dc0, ss, L, B, d, n_dir,
                                                     alpha, st, (flags & SRU_FLAG_V_ZERO) != 0);
    } else {
        // one (U type, dU type, channel width) instantiation per combination
        auto run = [&](auto ut, auto dut, auto cjc) {
            using UT = decltype(ut);
            using DUT = decltype(dut);
            return launch_bwd_seq<UT, DUT, decltype(cjc)::value>(mp, v, b, mask, ckpt, dc_T, dU, dx, partial, dc0,
                                                                 order_ws, L, B, d, n_dir, alpha, st);
        };
        using C64 = std::integral_constant<int, kSeqCJ>;
        const __nv_bfloat16 hb{};
        s = ub ? (db16 ? run(hb, hb, C64{}) : run(hb, 0.f, C64{})) : (db16 ? run(0.f, hb, C64{}) : run(0.f, 0.f, C64{}));
    }
    if (s != SRU_OK) return s;
    const int64_t rows = scan ? scan_chunks(L) * B : B;
    const size_t nred = (size_t)n_dir * 4 * d;
    sru::sru_reduce_dvdb_kernel<<<blocks_for(nred, sru::kRedCols), sru::kRedCols * sru::kRedSlices, 0, st>>>(
        partial, (int)rows, (int)d, n_dir, dv, db);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

sru_status sru_forward_scan_noalloc(const void* U, int u_t, const float* x, const float* b, const float* c0,
                                    const uint8_t* mask, int64_t L, int64_t B, int64_t d, float alpha,
                                    int bidirectional, float* h, float* c_T, void* stream) {
    sru_status s = check_layer_sizes(L, B, d);
    if (s != SRU_OK) return s;
    if (u_t != SRU_F32 && u_t != SRU_BF16) return SRU_ERR_INVALID;
    const int n_dir = bidirectional ? 2 : 1;
    if (B == 0) return SRU_OK;
    if (!b || !c_T) return SRU_ERR_INVALID;
    if (!aligned8_or_null(b) || !aligned8_or_null(c0) || !aligned8_or_null(c_T)) return SRU_ERR_INVALID;
    if (L > 0 && (!U || !x || !h || !aligned16(U) || !aligned16(x) || !aligned16(h))) return SRU_ERR_INVALID;
    const int64_t items = scan_chunks(L) * ((d + sru::kRecCJ - 1) / sru::kRecCJ) * B * n_dir;
    size_t agg_a_off = 0, agg_b_off = 0, prefix_off = 0;
    if (noalloc_scan_bytes(items, &agg_a_off, &agg_b_off, &prefix_off) > kNoAllocScratchBytes)
        return SRU_ERR_UNSUPPORTED;  // larger than the static scratch
    cudaStream_t st = as_stream(stream);
    if (L == 0) {
        const size_t n = (size_t)B * n_dir * d;
        sru::sru_copy_state_kernel<<<blocks_for(n, 256), 256, 0, st>>>(c0, c_T, n);
        SRU_CUDA_TRY(cudaGetLastError());
        return SRU_OK;
    }
    void* scratch = nullptr;
    s = noalloc_scratch_address(st, &scratch);
    if (s != SRU_OK) return s;
    uint8_t* base = static_cast<uint8_t*>(scratch);
    sru::ScanState ss;
    ss.flags = reinterpret_cast<unsigned*>(base);
    ss.agg_a = reinterpret_cast<float*>(base + agg_a_off);
    ss.agg_b = reinterpret_cast<float*>(base + agg_b_off);
    ss.prefix = reinterpret_cast<float*>(base + prefix_off);
    ss.withhold = -1;
    RecMaps mp;
    if (!map_u_tensor(&mp.u, U, u_t, L, B, d, n_dir, sru::kRecCJ) || !map_f32_rows(&mp.x, x, L, B, d, sru::kRecCJ))
        return SRU_ERR_INVALID;
    if (u_t == SRU_BF16)
        return launch_fwd_scan<__nv_bfloat16>(mp, b, c0, mask, h, c_T, nullptr, ss, L, B, d, n_dir, alpha, st);
    return launch_fwd_scan<float>(mp, b, c0, mask, h, c_T, nullptr, ss, L, B, d, n_dir, alpha, st);
}

sru_status sru_forward_fused(const void* X, const void* W, const float* x, const float* v, const float* b,
                             const float* c0, const uint8_t* mask, int64_t L, int64_t B, int64_t d, float alpha,
                             int bidirectional, float* h, float* c_T, void* U, void* workspace,
                             size_t workspace_bytes, void* stream) {
    sru_status s = check_layer_sizes(L, B, d);
    if (s != SRU_OK) return s;
    const int n_dir = bidirectional ? 2 : 1;
    if (B == 0) return SRU_OK;
    if (!v || !b || !c_T) return SRU_ERR_INVALID;
    if (!aligned8_or_null(v) || !aligned8_or_null(b) || !aligned8_or_null(c0) || !aligned8_or_null(c_T))
        return SRU_ERR_INVALID;
    cudaStream_t st = as_stream(stream);
    if (L == 0) {
        const size_t n = (size_t)B * n_dir * d;
        sru::sru_copy_state_kernel<<<blocks_for(n, 256), 256, 0, st>>>(c0, c_T, n);
        SRU_CUDA_TRY(cudaGetLastError());
        return SRU_OK;
    }
    if (!X || !W || !x || !h || !workspace) return SRU_ERR_INVALID;
    if (!aligned16(X) || !aligned16(W) || !aligned16(x) || !aligned16(h) || !aligned16(workspace) ||
        (U && !aligned16(U)))
        return SRU_ERR_INVALID;
    const WsLayout w = ws_layout(L, B, d, n_dir, SRU_FLAG_FORCE_SEQUENTIAL);  // the smallest layout
    if (workspace_bytes < w.total) return SRU_ERR_INVALID;
    CUtensorMap mx, mw, mu;
    {
        const uint64_t dims[3] = {(uint64_t)d, (uint64_t)B, (uint64_t)L};
        const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)B * d * 2};
        const uint32_t box[3] = {64, (uint32_t)sru::fused::kBb, (uint32_t)sru::fused::kTt};
        if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, X, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SRU_ERR_INVALID;
    }
    {
        const uint64_t dims[3] = {(uint64_t)d, (uint64_t)d, (uint64_t)(3 * n_dir)};
        const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)d * d * 2};
        // half a slice's 32 channels of all 3 gates
        const uint32_t box[3] = {64, (uint32_t)(sru::fused::kCh / 2), 3};
        if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, W, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SRU_ERR_INVALID;
    }
    std::memset(&mu, 0, sizeof(mu));
    if (U) {
        const uint64_t dims[5] = {(uint64_t)d, 3, (uint64_t)n_dir, (uint64_t)B, (uint64_t)L};
        const uint64_t strides[4] = {(uint64_t)d * 2, (uint64_t)3 * d * 2, (uint64_t)n_dir * 3 * d * 2,
                                     (uint64_t)B * n_dir * 3 * d * 2};
        const uint32_t box[5] = {(uint32_t)sru::fused::kCh, 3, 1, (uint32_t)sru::fused::kBb,
                                 (uint32_t)sru::fused::kTt};
        if (!make_map(&mu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, U, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SRU_ERR_INVALID;
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    sru::fused::FusedArgs fa;
    fa.x = x;
    fa.v = v;
    fa.bias = b;
    fa.c0 = c0;
    fa.mask = mask;
    fa.h = h;
    fa.c_T = c_T;
    fa.ckpt = U ? reinterpret_cast<float*>(ws + w.ckpt_off) : nullptr;
    fa.carry = reinterpret_cast<unsigned long long*>(ws + w.carry_off);
    fa.L = (int)L;
    fa.B = (int)B;
    fa.d = (int)d;
    fa.n_dir = n_dir;
    fa.alpha = alpha;
    fa.write_u = U != nullptr;
    SRU_CUDA_TRY(cudaMemsetAsync(fa.carry, 0, (size_t)B * n_dir * d * sizeof(unsigned long long), st));
    const int64_t nT = (L + sru::fused::kTt - 1) / sru::fused::kTt;
    const int64_t njs = (d + sru::fused::kCh - 1) / sru::fused::kCh;
    const int64_t nbgp = (B + 2 * sru::fused::kBb - 1) / (2 * sru::fused::kBb);
    const int64_t items = nT * n_dir * nbgp * njs;
    if (items >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
    const void* kern = reinterpret_cast<const void*>(sru::fused::sru_fused_fwd_kernel);
    SRU_CUDA_TRY(ensure_smem(kern, sru::fused::kSmemBytes));
    const int64_t max_pairs = fused_resident_pairs();
    if (max_pairs < 1) return cuda_fail(cudaErrorLaunchOutOfResources);
    const int64_t pairs = items < max_pairs ? items : max_pairs;
    sru::fused::sru_fused_fwd_kernel<<<(unsigned)(2 * pairs), sru::fused::kThreads, sru::fused::kSmemBytes, st>>>(
        mx, mw, mu, fa);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

// Split-K for fp32 products with fewer output tiles than CTA pairs and a long
// reduction (the weight gradients dW = dU^T X of narrow layers): k part s of
// every tile is written to slab s of a scratch buffer (rows s * R_pad ..,
// R_pad = R rounded up to whole tiles), then splitk_reduce_kernel sums the
// slabs in order into the output, so the result is the same bits every run.
// S comes from a time model measured on B200: a round of units costs
// kper k-blocks at 0.35 us each plus 2 us of fill and epilogue, and the slabs
// cost their bytes twice (written, then read by the sum) at 5 TB/s plus 3 us
// for the sum's launch; S = 1 means no split pays.
struct SplitPlan {
    int64_t splits, slab_rows;
    size_t bytes;
};
static SplitPlan split_plan(int64_t R, int64_t C, int64_t Kr) {
    constexpr double kKblockUs = 0.35, kUnitUs = 2.0, kSlabBytesPerUs = 5.0e6, kSumUs = 3.0;
    const int64_t P = sm_count() / 2;
    const int64_t tiles = ((R + sru::gemm::P_BM - 1) / sru::gemm::P_BM) * ((C + sru::gemm::P_BN - 1) / sru::gemm::P_BN);
    const int64_t kblocks = (Kr + sru::gemm::BK - 1) / sru::gemm::BK;
    SplitPlan pl{1, ((R + sru::gemm::P_BM - 1) / sru::gemm::P_BM) * sru::gemm::P_BM, 0};
    auto model_us = [&](int64_t S) {
        const int64_t kper = (kblocks + S - 1) / S;
        const double slabs = S > 1 ? (double)S * pl.slab_rows * C * 4 * 2 / kSlabBytesPerUs + kSumUs : 0.0;
        return (double)((tiles * S + P - 1) / P) * (kper * kKblockUs + kUnitUs) + slabs;
    };
    double best = model_us(1);
    for (int64_t S0 = 2; S0 <= 32 && S0 * 4 <= kblocks; ++S0) {
        // the kernel gives part s the k-blocks [s kper, (s + 1) kper) with kper =
        // ceil(kblocks / S): take S so that no part is empty (an empty part would
        // store an accumulator no MMA wrote)
        const int64_t S = (kblocks + (kblocks + S0 - 1) / S0 - 1) / ((kblocks + S0 - 1) / S0);
        const double t = model_us(S);
        if (t < best) {
            best = t;
            pl.splits = S;
        }
    }
    pl.bytes = pl.splits > 1 ? (size_t)pl.splits * pl.slab_rows * C * 4 : 0;
    return pl;
}
// dW[N, K] = dU[M, N]^T X[M, K] (bf16 operands, fp32 output) with the split
// plan above when `scratch` holds its slabs, else as sru_project_backward does.
static sru_status project_dW_split(const void* dU, const void* X, float* dW, int64_t M, int64_t N, int64_t K, void* scratch,
                            size_t scratch_bytes, cudaStream_t st) {
    if (M == 0) return zero_f32(dW, (size_t)N * K, st);
    CUtensorMap ma, mb;
    if (!map_mnmajor(&ma, dU, N, M, N) || !map_mnmajor(&mb, X, K, M, K)) return SRU_ERR_INVALID;
    const SplitPlan pl = split_plan(N, K, M);
    if (pl.splits <= 1 || scratch == nullptr || scratch_bytes < pl.bytes)
        return launch_tc_gemm<true, true, sru::gemm::kOutF32>(ma, mb, dW, N, K, M, st, 1, -1, /*tail_split=*/true);
    auto kern = sru::gemm::tc_gemm_pair_kernel<true, true, sru::gemm::kOutF32>;
    SRU_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kern), sru::gemm::P_SMEM_BYTES));
    CUtensorMap mo;
    {
        const uint64_t dims[2] = {(uint64_t)K, (uint64_t)(pl.slab_rows * pl.splits)};
        const uint64_t strides[1] = {(uint64_t)K * 4};
        const uint32_t box[2] = {(uint32_t)sru::gemm::EpiChunk<sru::gemm::kOutF32>::kCols, 32};
        if (!make_map(&mo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, scratch, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return SRU_ERR_INVALID;
    }
    const int64_t tiles = ((N + sru::gemm::P_BM - 1) / sru::gemm::P_BM) * ((K + sru::gemm::P_BN - 1) / sru::gemm::P_BN);
    const int64_t units = tiles * pl.splits;
    const int64_t pairs = units < sm_count() / 2 ? units : sm_count() / 2;
    kern<<<(unsigned)(2 * pairs), sru::gemm::THREADS, sru::gemm::P_SMEM_BYTES, st>>>(
        ma, mb, mo, (int)N, (int)K, (int)M, (int)pl.splits, 1, 0, (int)pl.slab_rows);
    SRU_CUDA_TRY(cudaGetLastError());
    const size_t n4 = (size_t)N * K / 4;
    sru::gemm::splitk_reduce_kernel<<<(unsigned)std::min<size_t>(blocks_for(n4, 256), (size_t)sm_count() * 8), 256, 0,
                                      st>>>(reinterpret_cast<const float4*>(scratch), reinterpret_cast<float4*>(dW),
                                            (int)N, (int)(K / 4), (int)pl.slab_rows, (int)pl.splits);
    SRU_CUDA_TRY(cudaGetLastError());
    return SRU_OK;
}

sru_status sru_project_factored(const void* X, const void* Wq, const void* Wo, void* P, void* U, int u_t,
                                int64_t M, int64_t N, int64_t K, int64_t Kp, void* stream) {
    if (M < 0 || N < 0 || K < 1 || Kp < 1) return SRU_ERR_INVALID;
    if (!X || !Wq || !Wo || !P || !U) return SRU_ERR_INVALID;
    if (u_t != SRU_BF16 && u_t != SRU_F32) return SRU_ERR_INVALID;
    if (K % 8 != 0 || Kp % 8 != 0 || N % 8 != 0) return SRU_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return SRU_OK;
    sru_status s = sru_project(X, SRU_BF16, Wq, SRU_BF16, P, SRU_BF16, M, Kp, K, stream);
    if (s != SRU_OK) return s;
    return sru_project(P, SRU_BF16, Wo, SRU_BF16, U, u_t, M, N, Kp, stream);
}

size_t sru_project_factored_backward_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t Kp) {
    if (M < 1 || N < 8 || K < 8 || Kp < 8 || N % 8 != 0 || K % 8 != 0 || Kp % 8 != 0) return 0;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) || Kp >= ((int64_t)1 << 31))
        return 0;
    return round256(std::max(split_plan(N, Kp, M).bytes, split_plan(Kp, K, M).bytes));
}

sru_status sru_project_factored_backward(const void* dU, const void* X, const void* Wq, const void* Wo,
                                         const void* P, void* dP, float* dX, int accumulate, float* dWq,
                                         float* dWo, int64_t M, int64_t N, int64_t K, int64_t Kp, void* workspace,
                                         size_t workspace_bytes, void* stream) {
    if (M < 0 || N < 1 || K < 1 || Kp < 1) return SRU_ERR_INVALID;
    if (!dU || !Wo || !dP || !aligned16(dU) || !aligned16(Wo) || !aligned16(dP)) return SRU_ERR_INVALID;
    if (workspace != nullptr && !aligned16(workspace)) return SRU_ERR_INVALID;
    if (dWo && (!P || !aligned16(P) || !aligned16(dWo))) return SRU_ERR_INVALID;
    if (dWq && (!X || !aligned16(X) || !aligned16(dWq))) return SRU_ERR_INVALID;
    if (dX && (!Wq || !aligned16(Wq) || !aligned16(dX))) return SRU_ERR_INVALID;
    if (K % 8 != 0 || Kp % 8 != 0 || N % 8 != 0) return SRU_ERR_UNSUPPORTED;
    if (M >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || K >= ((int64_t)1 << 31) || Kp >= ((int64_t)1 << 31))
        return SRU_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    if (M == 0) {
        if (dWo) { sru_status s = zero_f32(dWo, (size_t)N * Kp, st); if (s) return s; }
        if (dWq) return zero_f32(dWq, (size_t)Kp * K, st);
        return SRU_OK;
    }
    CUtensorMap ma, mb;
    // dWo = dU^T P (split along the tokens when its tiles cannot fill the GPU and
    // the workspace holds the slabs)
    if (dWo) {
        sru_status s = project_dW_split(dU, P, dWo, M, N, Kp, workspace, workspace_bytes, st);
        if (s != SRU_OK) return s;
    }
    // dP = dU Wo (bf16): A = dU K-major over n; B(c = kp, red = n) = Wo[n][kp] MN-major
    {
        if (!map_kmajor(&ma, dU, M, N, sru::gemm::P_CM) || !map_mnmajor(&mb, Wo, Kp, N, Kp)) return SRU_ERR_INVALID;
        sru_status s = launch_tc_gemm<false, true, sru::gemm::kOutBF16>(ma, mb, dP, M, Kp, N, st);
        if (s != SRU_OK) return s;
    }
    // dWq = dP^T X and dX (+)= dP Wq: the gradients of the first product
    sru_status s = sru_project_backward(dP, X, Wq, SRU_BF16, dX, accumulate, nullptr, M, Kp, K, stream);
    if (s != SRU_OK || !dWq) return s;
    return project_dW_split(dP, X, dWq, M, Kp, K, workspace, workspace_bytes, st);
}

// ---- SRU++ attention producer
// Batch rows are processed in groups of G: one batched launch each for the
// scores, the softmax and A; G bounds the scores and probabilities buffers.
constexpr size_t kAttnGroupBytes = (size_t)256 << 20;
int64_t attn_group(int64_t L, int64_t B) {
    const int64_t g = (int64_t)(kAttnGroupBytes / ((size_t)L * L * 6));
    return g < 1 ? 1 : (g > B ? B : g);
}
struct AttnWs {
    size_t q, kv, s, p, a, r, total;
};
AttnWs attn_ws(int64_t L, int64_t B, int64_t dp) {
    AttnWs w{};
    const int64_t M = L * B, G = attn_group(L, B);
    size_t off = 0;
    w.q = off;  off += round256((size_t)M * dp * 2);
    w.kv = off; off += round256((size_t)M * 2 * dp * 2);
    w.s = off;  off += round256((size_t)G * L * L * 4);
    w.p = off;  off += round256((size_t)G * L * L * 2);
    w.a = off;  off += round256((size_t)M * dp * 4);
    w.r = off;  off += round256((size_t)M * dp * 2);
    w.total = off;
    return w;
}

size_t sru_attention_workspace_bytes(int64_t L, int64_t B, int64_t dp) {
    if (L < 1 || B < 1 || dp < 8 || dp % 8 != 0 || L % 8 != 0) return 0;
    return attn_ws(L, B, dp).total;
}

sru_status sru_attention_project(const void* X, const void* Wq, const void* Wkv, const void* Wo, float alpha,
                                 const float* ln_gamma, const float* ln_beta, int causal, void* U, int u_t,
                                 int64_t L, int64_t B, int64_t d, int64_t dp, int64_t N, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    if (L < 1 || B < 1 || d < 1 || dp < 1 || N < 1) return SRU_ERR_INVALID;
    if (!X || !Wq || !Wkv || !Wo || !U || !workspace || !aligned16(workspace)) return SRU_ERR_INVALID;
    if ((ln_gamma == nullptr) != (ln_beta == nullptr)) return SRU_ERR_INVALID;
    if (ln_gamma != nullptr && (!aligned16(ln_gamma) || !aligned16(ln_beta))) return SRU_ERR_INVALID;
    if (u_t != SRU_BF16 && u_t != SRU_F32) return SRU_ERR_INVALID;
    if (d % 8 != 0 || dp % 8 != 0 || N % 8 != 0 || L % 8 != 0) return SRU_ERR_UNSUPPORTED;
    const int64_t M = L * B;
    if (M >= ((int64_t)1 << 31) || L > 65536) return SRU_ERR_UNSUPPORTED;
    const AttnWs w = attn_ws(L, B, dp);
    if (workspace_bytes < w.total) return SRU_ERR_INVALID;
    cudaStream_t st = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    __nv_bfloat16* Q = reinterpret_cast<__nv_bfloat16*>(ws + w.q);
    __nv_bfloat16* KV = reinterpret_cast<__nv_bfloat16*>(ws + w.kv);
    float* S = reinterpret_cast<float*>(ws + w.s);
    __nv_bfloat16* P = reinterpret_cast<__nv_bfloat16*>(ws + w.p);
    float* A = reinterpret_cast<float*>(ws + w.a);
    __nv_bfloat16* R = reinterpret_cast<__nv_bfloat16*>(ws + w.r);
    // Q = X Wq^T, then [K | V] = Q [Wk; Wv]^T
    sru_status s = sru_project(X, SRU_BF16, Wq, SRU_BF16, Q, SRU_BF16, M, dp, d, stream);
    if (s != SRU_OK) return s;
    s = sru_project(Q, SRU_BF16, Wkv, SRU_BF16, KV, SRU_BF16, M, 2 * dp, dp, stream);
    if (s != SRU_OK) return s;
    const float scale = 1.0f / sqrtf((float)dp);
    const int64_t G = attn_group(L, B);
    // batch row b's tokens are rows t*B + b of the time-major Q, K, V and A
    for (int64_t b0 = 0; b0 < B; b0 += G) {
        const int64_t g = B - b0 < G ? B - b0 : G;
        CUtensorMap ma, mb;
        // S_z = Q_z K_z^T (z = 0 .. g-1): K-major over d'; batch stride d' / 2d', row stride B d' / 2B d'
        if (!map_kmajor_b(&ma, Q + b0 * dp, L, dp, B * dp, g, dp, sru::gemm::P_CM, 1) ||
            !map_kmajor_b(&mb, KV + b0 * 2 * dp, L, dp, B * 2 * dp, g, 2 * dp, kGemmBRows, 1))
            return SRU_ERR_INVALID;
        s = causal ? launch_tc_gemm_batched<false, false, sru::gemm::kOutF32, 1, 1, 1>(ma, mb, S, L, L, dp, L, g, L * L, st)
                   : launch_tc_gemm_batched<false, false, sru::gemm::kOutF32, 1, 1>(ma, mb, S, L, L, dp, L, g, L * L, st);
        if (s != SRU_OK) return s;
        s = launch_softmax_rows(S, P, L, g * L, scale, causal ? 1 : 0, st);
        if (s != SRU_OK) return s;
        // A_z = P_z V_z: P_z K-major over s (batch outermost); V_z(c = j, red = s) at
        // KV[(s*B + b0 + z)*2d' + d' + j]: MN-major, batch stride 2d'
        if (!map_kmajor_b(&ma, P, L, L, L, g, L * L, sru::gemm::P_CM, 2) ||
            !map_mnmajor_b(&mb, KV + b0 * 2 * dp + dp, dp, L, B * 2 * dp, g, 2 * dp, 1))
            return SRU_ERR_INVALID;
        s = causal ? launch_tc_gemm_batched<false, true, sru::gemm::kOutF32, 2, 1, 2>(ma, mb, A + b0 * dp, L, dp, L,
                                                                                     B * dp, g, dp, st)
                   : launch_tc_gemm_batched<false, true, sru::gemm::kOutF32, 2, 1>(ma, mb, A + b0 * dp, L, dp, L, B * dp,
                                                                                 g, dp, st);
        if (s != SRU_OK) return s;
    }
    s = launch_residual_norm(Q, A, alpha, ln_gamma, ln_beta, R, M, dp, st);
    if (s != SRU_OK) return s;
    return sru_project(R, SRU_BF16, Wo, SRU_BF16, U, u_t, M, N, dp, stream);
}

// ------------------------------------------------- attention producer backward
// Batch rows per group of the backward: scores / their gradient (fp32), P and
// dS (bf16) of one group stay under the same budget as the forward's.
static int64_t attn_bwd_group(int64_t L, int64_t B) {
    const int64_t g = (int64_t)(kAttnGroupBytes / ((size_t)L * L * 8));
    return g < 1 ? 1 : (g > B ? B : g);
}
struct AttnBwdWs {
    size_t dr, dq, dqa, da, dkv, dqb, s, p, ds, stats, part, split, split_bytes, total;
    bool fwd_p;  // the forward's workspace holds every batch row's probabilities (one group)
};
static AttnBwdWs attn_bwd_ws(int64_t L, int64_t B, int64_t d, int64_t dp, int64_t N) {
    AttnBwdWs w{};
    const int64_t M = L * B, G = attn_bwd_group(L, B);
    // slabs of the split-K weight gradients dWo (N x d'), dWkv (2d' x d'), dWq (d' x d)
    w.split_bytes = std::max(split_plan(N, dp, M).bytes, std::max(split_plan(2 * dp, dp, M).bytes,
                                                                  split_plan(dp, d, M).bytes));
    w.fwd_p = attn_group(L, B) >= B;
    size_t off = 0;
    w.dr = off;    off += round256((size_t)M * dp * 4);
    w.dq = off;    off += round256((size_t)M * dp * 4);
    w.dqa = off;   off += round256((size_t)M * dp * 4);
    w.da = off;    off += round256((size_t)M * dp * 2);
    w.dkv = off;   off += round256((size_t)M * 2 * dp * 2);
    w.dqb = off;   off += round256((size_t)M * dp * 2);
    w.s = off;     off += round256((size_t)G * L * L * 4);
    w.p = off;     off += w.fwd_p ? 0 : round256((size_t)G * L * L * 2);
    w.ds = off;    off += round256((size_t)G * L * L * 2);
    w.stats = off; off += round256((size_t)M * 8);
    w.part = off;  off += round256((size_t)((M + sru::kNormRows - 1) / sru::kNormRows) * 2 * dp * 4);
    w.split = off; off += round256(w.split_bytes);
    w.total = off;
    return w;
}

size_t sru_attention_backward_workspace_bytes(int64_t L, int64_t B, int64_t d, int64_t dp, int64_t N) {
    if (L < 1 || B < 1 || d < 8 || dp < 8 || N < 8 || d % 8 != 0 || dp % 8 != 0 || N % 8 != 0 || L % 8 != 0)
        return 0;
    if (L * B >= ((int64_t)1 << 31) || L > 65536) return 0;
    return attn_bwd_ws(L, B, d, dp, N).total;
}

sru_status sru_attention_project_backward(const void* dU, const void* X, const void* Wq, const void* Wkv,
                                          const void* Wo, float alpha, const float* ln_gamma,
                                          const float* ln_beta, int causal, const void* fwd_workspace,
                                          size_t fwd_workspace_bytes, float* dX, int accumulate, float* dWq,
                                          float* dWkv, float* dWo, float* dgamma, float* dbeta, int64_t L,
                                          int64_t B, int64_t d, int64_t dp, int64_t N, void* workspace,
                                          size_t workspace_bytes, void* stream) {
    if (L < 1 || B < 1 || d < 1 || dp < 1 || N < 1) return SRU_ERR_INVALID;
    if (!dU || !X || !Wq || !Wkv || !Wo || !fwd_workspace || !dX || !dWq || !dWkv || !dWo || !workspace)
        return SRU_ERR_INVALID;
    if (!aligned16(dU) || !aligned16(X) || !aligned16(Wq) || !aligned16(Wkv) || !aligned16(Wo) ||
        !aligned16(fwd_workspace) || !aligned16(dX) || !aligned16(dWq) || !aligned16(dWkv) || !aligned16(dWo) ||
        !aligned16(workspace))
        return SRU_ERR_INVALID;
    if ((ln_gamma == nullptr) != (ln_beta == nullptr)) return SRU_ERR_INVALID;
    if (ln_gamma != nullptr && (!aligned16(ln_gamma) || !aligned16(ln_beta))) return SRU_ERR_INVALID;
    const bool norm = ln_gamma != nullptr;
    if (norm && (!dgamma || !dbeta)) return SRU_ERR_INVALID;
    if (d % 8 != 0 || dp % 8 != 0 || N % 8 != 0 || L % 8 != 0) return SRU_ERR_UNSUPPORTED;
    const int64_t M = L * B;
    if (M >= ((int64_t)1 << 31) || L > 65536) return SRU_ERR_UNSUPPORTED;
    const AttnWs fw = attn_ws(L, B, dp);
    const AttnBwdWs w = attn_bwd_ws(L, B, d, dp, N);
    if (fwd_workspace_bytes < fw.total || workspace_bytes < w.total) return SRU_ERR_INVALID;
    cudaStream_t st = as_stream(stream);
    const uint8_t* fws = static_cast<const uint8_t*>(fwd_workspace);
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(fws + fw.q);
    const __nv_bfloat16* KV = reinterpret_cast<const __nv_bfloat16*>(fws + fw.kv);
    const float* A = reinterpret_cast<const float*>(fws + fw.a);
    const __nv_bfloat16* R = reinterpret_cast<const __nv_bfloat16*>(fws + fw.r);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* dR = reinterpret_cast<float*>(ws + w.dr);
    float* dQ = reinterpret_cast<float*>(ws + w.dq);
    float* dQa = reinterpret_cast<float*>(ws + w.dqa);
    __nv_bfloat16* dA = reinterpret_cast<__nv_bfloat16*>(ws + w.da);
    __nv_bfloat16* dKV = reinterpret_cast<__nv_bfloat16*>(ws + w.dkv);
    __nv_bfloat16* dQb = reinterpret_cast<__nv_bfloat16*>(ws + w.dqb);
    float* S = reinterpret_cast<float*>(ws + w.s);
    // with one group the forward's probabilities of every batch row are still in its workspace
    const __nv_bfloat16* Pf = reinterpret_cast<const __nv_bfloat16*>(fws + fw.p);
    __nv_bfloat16* P = w.fwd_p ? nullptr : reinterpret_cast<__nv_bfloat16*>(ws + w.p);
    __nv_bfloat16* dS = reinterpret_cast<__nv_bfloat16*>(ws + w.ds);
    float2* stats = reinterpret_cast<float2*>(ws + w.stats);
    float* part = reinterpret_cast<float*>(ws + w.part);
    void* split = ws + w.split;

    // U = R Wo^T:  dR = dU Wo,  dWo = dU^T R
    sru_status s = sru_project_backward(dU, R, Wo, SRU_BF16, dR, 0, nullptr, M, N, dp, stream);
    if (s != SRU_OK) return s;
    s = project_dW_split(dU, R, dWo, M, N, dp, split, w.split_bytes, st);
    if (s != SRU_OK) return s;
    // through the norm (or the identity): dQ = dZ, dA = alpha dZ.  With the norm, the
    // first stage of dgamma / dbeta (slices of kNormRows tokens) is taken inside the
    // norm's backward where the row fits in registers.
    const int64_t nv = (dp + 127) / 128;
    unsigned slices = (unsigned)((M + sru::kNormRows - 1) / sru::kNormRows);
    if (norm && nv <= 8) {
        auto run = nv <= 1 ? norm_backward_params_reg<1>
                   : nv <= 2 ? norm_backward_params_reg<2>
                   : nv <= 4 ? norm_backward_params_reg<4>
                             : norm_backward_params_reg<8>;
        slices = run(dR, Q, A, alpha, ln_gamma, dQ, dA, stats, part, M, dp, st);
        SRU_CUDA_TRY(cudaGetLastError());
    } else {
        s = launch_norm_backward(dR, Q, A, alpha, ln_gamma, dQ, dA, stats, M, dp, st);
        if (s != SRU_OK) return s;
        if (norm) {
            if (slices > 65535u) return SRU_ERR_UNSUPPORTED;
            const dim3 grid(blocks_for((size_t)dp, sru::kNormParamThreads), slices);
            sru::sru_norm_param_partial_kernel<<<grid, sru::kNormParamThreads, 0, st>>>(dR, Q, A, alpha, stats,
                                                                                       part, (int)M, (int)dp);
            SRU_CUDA_TRY(cudaGetLastError());
        }
    }
    if (norm) {
        sru::sru_norm_param_reduce_kernel<<<blocks_for((size_t)(2 * dp), sru::kNormRedCols),
                                            sru::kNormRedCols * sru::kNormRedGroups, 0, st>>>(part, (int)slices,
                                                                                            (int)dp, dgamma, dbeta);
        SRU_CUDA_TRY(cudaGetLastError());
    }
    const float scale = 1.0f / sqrtf((float)dp);
    const int64_t G = attn_bwd_group(L, B);
    // batch row b's tokens are rows t*B + b of the time-major Q, K, V, dA, dQ and [dK | dV]
    for (int64_t b0 = 0; b0 < B; b0 += G) {
        const int64_t g = B - b0 < G ? B - b0 : G;
        CUtensorMap ma, mb;
        // the forward's probabilities of this group: still in the forward's workspace
        // (one group there), else recomputed: S = Q K^T, softmax
        const __nv_bfloat16* Pg = w.fwd_p ? Pf + b0 * L * L : P;
        if (!w.fwd_p) {
            if (!map_kmajor_b(&ma, Q + b0 * dp, L, dp, B * dp, g, dp, sru::gemm::P_CM, 1) ||
                !map_kmajor_b(&mb, KV + b0 * 2 * dp, L, dp, B * 2 * dp, g, 2 * dp, kGemmBRows, 1))
                return SRU_ERR_INVALID;
            s = causal ? launch_tc_gemm_batched<false, false, sru::gemm::kOutF32, 1, 1, 1>(ma, mb, S, L, L, dp, L, g,
                                                                                          L * L, st)
                       : launch_tc_gemm_batched<false, false, sru::gemm::kOutF32, 1, 1>(ma, mb, S, L, L, dp, L, g,
                                                                                       L * L, st);
            if (s != SRU_OK) return s;
            s = launch_softmax_rows(S, P, L, g * L, scale, causal ? 1 : 0, st);
            if (s != SRU_OK) return s;
        }
        // dP = dA V^T (into S), then dS
        if (!map_kmajor_b(&ma, dA + b0 * dp, L, dp, B * dp, g, dp, sru::gemm::P_CM, 1) ||
            !map_kmajor_b(&mb, KV + b0 * 2 * dp + dp, L, dp, B * 2 * dp, g, 2 * dp, kGemmBRows, 1))
            return SRU_ERR_INVALID;
        s = causal ? launch_tc_gemm_batched<false, false, sru::gemm::kOutF32, 1, 1, 1>(ma, mb, S, L, L, dp, L, g, L * L, st)
                   : launch_tc_gemm_batched<false, false, sru::gemm::kOutF32, 1, 1>(ma, mb, S, L, L, dp, L, g, L * L, st);
        if (s != SRU_OK) return s;
        s = launch_softmax_backward_rows(S, Pg, dS, L, g * L, scale, causal ? 1 : 0, st);
        if (s != SRU_OK) return s;
        // dV = P^T dA and dK = dS^T Q (bf16, into [dK | dV]): the first operand read
        // MN-major (element (s, t) of batch z at z L^2 + t L + s), the second too
        // (element (j, t) at (t B + b0 + z) d' + j)
        __nv_bfloat16* dK0 = dKV + b0 * 2 * dp;
        if (!map_mnmajor_b(&ma, Pg, L, L, L, g, L * L, 2) || !map_mnmajor_b(&mb, dA + b0 * dp, dp, L, B * dp, g, dp, 1))
            return SRU_ERR_INVALID;
        s = causal ? launch_tc_gemm_batched<true, true, sru::gemm::kOutBF16, 2, 1, 3>(ma, mb, dK0 + dp, L, dp, L,
                                                                                     B * 2 * dp, g, 2 * dp, st)
                   : launch_tc_gemm_batched<true, true, sru::gemm::kOutBF16, 2, 1>(ma, mb, dK0 + dp, L, dp, L,
                                                                                  B * 2 * dp, g, 2 * dp, st);
        if (s != SRU_OK) return s;
        if (!map_mnmajor_b(&ma, dS, L, L, L, g, L * L, 2) || !map_mnmajor_b(&mb, Q + b0 * dp, dp, L, B * dp, g, dp, 1))
            return SRU_ERR_INVALID;
        s = causal ? launch_tc_gemm_batched<true, true, sru::gemm::kOutBF16, 2, 1, 3>(ma, mb, dK0, L, dp, L,
                                                                                     B * 2 * dp, g, 2 * dp, st)
                   : launch_tc_gemm_batched<true, true, sru::gemm::kOutBF16, 2, 1>(ma, mb, dK0, L, dp, L, B * 2 * dp,
                                                                                  g, 2 * dp, st);
        if (s != SRU_OK) return s;
        // dS K (into dQa, added to dQ below): dS K-major over s; K (c = j, red = s) at
        // KV[(s B + b0 + z) 2d' + j]: MN-major
        if (!map_kmajor_b(&ma, dS, L, L, L, g, L * L, sru::gemm::P_CM, 2) ||
            !map_mnmajor_b(&mb, KV + b0 * 2 * dp, dp, L, B * 2 * dp, g, 2 * dp, 1))
            return SRU_ERR_INVALID;
        s = causal ? launch_tc_gemm_batched<false, true, sru::gemm::kOutF32, 2, 1, 2>(ma, mb, dQa + b0 * dp, L, dp, L,
                                                                                     B * dp, g, dp, st)
                   : launch_tc_gemm_batched<false, true, sru::gemm::kOutF32, 2, 1>(ma, mb, dQa + b0 * dp, L, dp, L,
                                                                                  B * dp, g, dp, st);
        if (s != SRU_OK) return s;
    }
    // [K | V] = Q Wkv^T:  dQ += [dK | dV] Wkv,  dWkv = [dK | dV]^T Q
    s = sru_project_backward(dKV, Q, Wkv, SRU_BF16, dQ, 1, nullptr, M, 2 * dp, dp, stream);
    if (s != SRU_OK) return s;
    s = project_dW_split(dKV, Q, dWkv, M, 2 * dp, dp, split, w.split_bytes, st);
    if (s != SRU_OK) return s;
    // Q = X Wq^T:  dWq = dQ^T X,  dX (+)= dQ Wq  (dQ = dZ + [dK | dV] Wkv + dS K rounded to
    // bf16 as the products' operand)
    const size_t n4 = (size_t)M * dp / 4;
    sru::sru_add_to_bf16_kernel<<<(unsigned)std::min<size_t>(blocks_for(n4, 256), (size_t)sm_count() * 8), 256, 0,
                                  st>>>(reinterpret_cast<const float4*>(dQ), reinterpret_cast<const float4*>(dQa),
                                        reinterpret_cast<uint2*>(dQb), n4);
    SRU_CUDA_TRY(cudaGetLastError());
    s = sru_project_backward(dQb, X, Wq, SRU_BF16, dX, accumulate, nullptr, M, dp, d, stream);
    if (s != SRU_OK) return s;
    return project_dW_split(dQb, X, dWq, M, dp, d, split, w.split_bytes, st);
}

// Batch rows from which the step's product runs on the tensor cores (measured:
// the fused CUDA-core kernel's registers per channel grow with B).
constexpr int64_t kDecodeTensorMinB = 8;

// (B a multiple of 8: u's rows, B floats each, are a tensor-core output whose
// row pitch must be a multiple of 16 bytes)
bool decode_tensor_path(int64_t B) { return B >= kDecodeTensorMinB && B % 8 == 0; }

size_t sru_decode_workspace_bytes(int64_t B, int64_t d) {
    if (!decode_tensor_path(B) || d < 1) return 0;
    return round256((size_t)3 * d * B * sizeof(float));
}

sru_status sru_decode_step(const void* X_t, const void* W, const float* x_t, const float* v, const float* b,
                           float* c, float* h_t, int64_t B, int64_t d, float alpha, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (B < 0 || d < 1) return SRU_ERR_INVALID;
    if (d % 8 != 0) return SRU_ERR_UNSUPPORTED;
    if (B == 0) return SRU_OK;
    if (!X_t || !W || !x_t || !v || !b || !c || !h_t) return SRU_ERR_INVALID;
    if (!aligned16(X_t) || !aligned16(W) || !aligned16(x_t) || !aligned16(c) || !aligned16(h_t))
        return SRU_ERR_INVALID;
    if (d > ((int64_t)1 << 24) || B > ((int64_t)1 << 20)) return SRU_ERR_UNSUPPORTED;
    if (workspace != nullptr && decode_tensor_path(B)) {
        // u = W_cat X_t^T (3d x B) on the tensor cores, then the cell update
        if (!aligned16(workspace) || workspace_bytes < sru_decode_workspace_bytes(B, d)) return SRU_ERR_INVALID;
        if (3 * d >= ((int64_t)1 << 31)) return SRU_ERR_UNSUPPORTED;
        float* u = static_cast<float*>(workspace);
        sru_status s = sru_project(W, SRU_BF16, X_t, SRU_BF16, u, SRU_F32, 3 * d, B, d, stream);
        if (s != SRU_OK) return s;
        const size_t n = (size_t)B * d;
        sru::sru_decode_cell_kernel<<<blocks_for(n, 256), 256, 0, as_stream(stream)>>>(u, x_t, v, b, c, h_t, (int)B,
                                                                                        (int)d, alpha);
        SRU_CUDA_TRY(cudaGetLastError());
        return SRU_OK;
    }
    const int nb = decode_rows_per_pass(B);
    if ((B + nb - 1) / nb > 65535) return SRU_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    switch (nb) {
        case 1: return launch_decode_nb<1>(X_t, W, x_t, v, b, c, h_t, B, d, alpha, st);
        case 2: return launch_decode_nb<2>(X_t, W, x_t, v, b, c, h_t, B, d, alpha, st);
        case 4: return launch_decode_nb<4>(X_t, W, x_t, v, b, c, h_t, B, d, alpha, st);
        case 8: return launch_decode_nb<8>(X_t, W, x_t, v, b, c, h_t, B, d, alpha, st);
        default: return launch_decode_nb<16>(X_t, W, x_t, v, b, c, h_t, B, d, alpha, st);
    }
}

sru_status sru_sync_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned word = 0;
    e = cudaMemcpyFromSymbol(&word, sru::g_error_word, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word != 0) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(sru::g_error_word, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e);
        return SRU_ERR_TIMEOUT;
    }
    return SRU_OK;
}

}  // extern "C"
