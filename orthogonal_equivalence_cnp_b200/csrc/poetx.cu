// libpoetx: C ABI of the POET-X layer (see include/poetx.h for the contract of every call).
//
// Single translation unit: the kernels live in the included headers.  This file holds the
// host side: argument validation, workspace planning, TMA tensor-map encoding, and the
// orchestration of the input-centric chain (replication review of POET-X, "Summary").
#include <algorithm>
#include <atomic>
#include <utility>
#include <vector>
#include <initializer_list>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/poetx_testing.h"
#include "common.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "sm100.cuh"
#include "cnp_onchip.cuh"

using namespace poetx;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kNumSms = 148;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int esize(int dt) { return dt == BF16 ? 2 : 4; }

// Sequential carve-out of the caller's workspace (offsets only; nothing is allocated).
struct Plan {
  size_t total = 0;
  size_t take(size_t bytes) {
    size_t o = total;
    total += align256(bytes);
    return o;
  }
};

#define POETX_TRY(expr)                  \
  do {                                   \
    poetx_status _s = (expr);            \
    if (_s != POETX_OK) return _s;       \
  } while (0)

// Opts a kernel into `smem` bytes of dynamic shared memory and the largest shared-memory carveout
// (the default carveout can leave room for fewer resident blocks than the shared memory allows).
template <typename K>
inline bool set_smem(K kern, size_t smem) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess &&
         cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess;
}

inline poetx_status last_launch() {
  return cudaGetLastError() == cudaSuccess ? POETX_OK : POETX_ERR_CUDA;
}

// ------------------------------------------------------------------ launch accounting
// Every kernel launch of the library goes through a LaunchScope: it counts the launch and, when
// profiling is on, brackets it with a CUDA event pair on the launching stream.
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> recs;
  std::atomic<unsigned long long> launches{0};
  cudaEvent_t take() {
    if (used == pool.size()) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
      pool.push_back(e);
    }
    return pool[used++];
  }
};
Profiler& prof() {
  static Profiler* p = new Profiler();  // never destroyed: events may outlive static teardown
  return *p;
}

struct LaunchScope {
  int cls;
  cudaStream_t st;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  unsigned int flags = cudaEventRecordDefault;
  LaunchScope(int c, cudaStream_t s) : cls(c), st(s) {
    Profiler& p = prof();
    p.launches.fetch_add(1, std::memory_order_relaxed);
    if (p.on) {
      std::lock_guard<std::mutex> g(p.mu);
      e0 = p.take();
      e1 = p.take();
      // Under stream capture the records must be external so that they become event nodes.
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      cudaStreamIsCapturing(st, &cs);
      flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
      if (e0 && e1) cudaEventRecordWithFlags(e0, st, flags);
    }
  }
  ~LaunchScope() {
    if (e0 && e1) {
      Profiler& p = prof();
      cudaEventRecordWithFlags(e1, st, flags);
      std::lock_guard<std::mutex> g(p.mu);
      p.recs.push_back({cls, {e0, e1}});
    }
  }
};

// Launch with a programmatic dependency on the previous kernel of the stream: the kernel may
// be scheduled while that one finishes and waits for it in griddep_wait() before touching its
// results (every kernel of this library does).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_prio(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool high,
                            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (high) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess) {
      attr[1].id = cudaLaunchAttributePriority;
      attr[1].val.priority = greatest;
      cfg.numAttrs = 2;
    }
  }
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  return launch_pdl_prio(kern, grid, block, smem, st, false, args...);
}

poetx_status check_desc(const poetx_desc* d) {
  if (d == nullptr) return POETX_ERR_INVALID_ARG;
  if (d->dtype != POETX_F32 && d->dtype != POETX_BF16) return POETX_ERR_INVALID_ARG;
  if (d->mode != POETX_FAST && d->mode != POETX_MEM) return POETX_ERR_INVALID_ARG;
  if (d->d_in <= 0 || d->d_out <= 0 || d->b <= 0 || d->k < 0) return POETX_ERR_INVALID_ARG;
  const int b = d->b;
  if (b != 32 && b != 64 && b != 128 && b != 256 && b != 512) return POETX_ERR_UNSUPPORTED_SHAPE;
  if (d->dtype == POETX_BF16 && b < 64) return POETX_ERR_UNSUPPORTED_SHAPE;
  if (d->k > 8) return POETX_ERR_UNSUPPORTED_SHAPE;
  if (d->d_in % b != 0 || d->d_out % b != 0) return POETX_ERR_UNSUPPORTED_SHAPE;
  // The permutation kernel stages up to three feature rows (d * element size each) in one
  // block's shared memory: at most 64 KiB per row.
  const int dmax = d->dtype == POETX_BF16 ? 32768 : 16384;
  if (d->d_in > dmax || d->d_out > dmax) return POETX_ERR_UNSUPPORTED_SHAPE;
  return POETX_OK;
}

// ------------------------------------------------------------------------------ GEMM dispatch
// Checks that every element a GEMM may address lies inside its arrays (the tensor-core path
// relies on TMA zero-fill beyond the array extent; the SIMT path masks m < M, n < N, k < K).
bool view_fits(const Operand& op, bool mn, long mnext, long kext, long batch) {
  if (op.base == nullptr || op.ld < op.cols || op.rows <= 0 || op.cols <= 0) return false;
  const long r_last = (batch - 1) * op.zrow + (mn ? kext : mnext);
  const long c_last = (batch - 1) * op.zcol + (mn ? mnext : kext);
  return r_last <= op.rows && c_last <= op.cols;
}

poetx_status check_gemm(const GemmDesc& g, int dt) {
  if (g.M <= 0 || g.N <= 0 || g.K < 0 || g.batch <= 0 || g.splits <= 0) return POETX_ERR_INVALID_ARG;
  if (g.batch * (long)g.splits > 65535) return POETX_ERR_UNSUPPORTED_SHAPE;
  if (g.K > 0) {
    if (!view_fits(g.A, g.a_mn, g.M, g.K, g.batch)) return POETX_ERR_INVALID_ARG;
    if (!view_fits(g.B, g.b_mn, g.N, g.K, g.batch)) return POETX_ERR_INVALID_ARG;
  }
  if (dt == BF16) {
    // Tensor-core path: N in whole 64-column tiles, 16-byte aligned rows and coordinates.
    if (g.N % 64 != 0) return POETX_ERR_UNSUPPORTED_SHAPE;
    const Operand* ops[2] = {&g.A, &g.B};
    for (const Operand* op : ops)
      if (!aligned16(op->base) || op->ld % 8 || op->zcol % 8) return POETX_ERR_ALIGNMENT;
    const Epilogue& e = g.epi;
    if (e.d1 && (!aligned16(e.d1) || e.ld1 % 8 || e.zcol1 % 8 || e.split_stride1 % 8)) return POETX_ERR_ALIGNMENT;
    if (e.red1 && (!e.d1 || e.d1_dtype != F32)) return POETX_ERR_INVALID_ARG;
    if (e.d2 && (!aligned16(e.d2) || e.ld2 % 4 || e.zcol2 % 4)) return POETX_ERR_ALIGNMENT;
    if (e.c && (!aligned16(e.c) || e.ldc % 8 || e.zcolc % 8)) return POETX_ERR_ALIGNMENT;
  }
  return POETX_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

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

// bf16 2-D tensor map over a whole operand array with a box of (inner x outer) elements and
// 128-byte swizzle; reads beyond the array extent return zeros.
Operand view(const void* base, long rows, long cols, long ld, long zrow = 0, long zcol = 0) {
  Operand o;
  o.base = base; o.rows = rows; o.cols = cols; o.ld = ld; o.zrow = zrow; o.zcol = zcol;
  return o;
}

// 2-D tensor map of a row-major bf16 (or fp32) array, 128-byte swizzle; box_inner elements must
// span 128 bytes (64 bf16 / 32 fp32).  Int8 codes (dt = U8) are mapped unswizzled (the
// converter warps read them row by row), any box up to 256 x 256.
bool make_tmap(CUtensorMap* m, const Operand& op, uint32_t box_inner, uint32_t box_outer, int dt = BF16) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const uint64_t es = dt == F32 ? 4 : dt == U8 ? 1 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)op.cols, (cuuint64_t)op.rows};
  cuuint64_t strides[1] = {(cuuint64_t)op.ld * es};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType type = dt == F32  ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : dt == U8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                              : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return fn(m, type, 2, const_cast<void*>(op.base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            dt == U8 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int ST, bool AMN, bool BMN>
poetx_status launch_tc(const GemmDesc& g, cudaStream_t st, int cls) {
  static bool attr_done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return POETX_ERR_CUDA;
  constexpr size_t smem = tc_smem_bytes<BN, ST>();
  auto kern = gemm_bf16_tc<BN, ST, AMN, BMN>;
  if (!attr_done[dev]) {
    if (!set_smem(kern, smem)) return POETX_ERR_CUDA;
    attr_done[dev] = true;
  }
  CUtensorMap ta, tb, td;
  if (!make_tmap(&ta, g.A, 64, AMN ? 64 : TC_BM)) return POETX_ERR_CUDA;
  if (!make_tmap(&tb, g.B, 64, BMN ? 64 : BN)) return POETX_ERR_CUDA;
  TcArgs a;
  a.M = g.M; a.N = g.N; a.K = g.K; a.splits = g.splits;
  a.a_zrow = (int)g.A.zrow; a.a_zcol = (int)g.A.zcol; a.b_zrow = (int)g.B.zrow; a.b_zcol = (int)g.B.zcol;
  a.epi = g.epi;
  a.b_early = g.b_static ? 1 : 0;
  // TMA-store epilogue for a plain bf16 result batched (if at all) along columns: the map spans
  // every batch's columns, boxes of 64 columns x 32 rows.
  const Epilogue& e = g.epi;
  a.tma_store = e.d1 != nullptr && e.d1_dtype == BF16 && e.alpha1 == 1.f && e.beta1 == 0.f && !e.c && !e.diag1 &&
                !e.d2 && !e.red1 && e.split_stride1 == 0 && e.zrow1 == 0 && g.splits == 1 && e.zcol1 % 8 == 0;
  if (a.tma_store) {
    if (!make_tmap(&td, view(e.d1, g.M, (long)(g.batch - 1) * e.zcol1 + g.N, e.ld1), 64, 32)) return POETX_ERR_CUDA;
  } else {
    td = ta;  // unused
  }
  dim3 grid(g.N / BN, (g.M + TC_BM - 1) / TC_BM, g.batch * g.splits);
  LaunchScope ls(cls, st);
  if (launch_pdl(kern, grid, dim3(128), smem, st, ta, tb, td, a) != cudaSuccess) return POETX_ERR_CUDA;
  return last_launch();
}

template <int BN, int ST>
poetx_status launch_tc_major(const GemmDesc& g, cudaStream_t st, int cls) {
  if (!g.a_mn && !g.b_mn) return launch_tc<BN, ST, false, false>(g, st, cls);
  if (!g.a_mn && g.b_mn) return launch_tc<BN, ST, false, true>(g, st, cls);
  if (g.a_mn && !g.b_mn) return launch_tc<BN, ST, true, false>(g, st, cls);
  return launch_tc<BN, ST, true, true>(g, st, cls);
}

poetx_status run_gemm(int dt, const GemmDesc& g, cudaStream_t st, int cls) {
  POETX_TRY(check_gemm(g, dt));
  if (dt == BF16) {
    // Long K (>= 16 k-tiles per CTA): deep ring, one CTA per SM, widest tile.  Short K: a
    // 96 KiB ring so two CTAs share an SM (one's epilogue overlaps the other's loads); the
    // full 256-column tile (A read once) as long as it still fills 1.5 CTAs per SM.
    const long kt = ((long)(g.K + TC_BK - 1) / TC_BK) / g.splits;
    const long base = (long)((g.M + TC_BM - 1) / TC_BM) * g.batch * g.splits;
    if (kt >= 16) {
      // The widest tile that still occupies three quarters of the SMs.
      if (g.N % 256 == 0 && 4 * base * (g.N / 256) >= 3 * kNumSms) return launch_tc_major<256, 4>(g, st, cls);
      if (g.N % 128 == 0 && 4 * base * (g.N / 128) >= 3 * kNumSms) return launch_tc_major<128, 6>(g, st, cls);
      return launch_tc_major<64, 8>(g, st, cls);
    }
    if (g.N % 256 == 0 && 2 * base * (g.N / 256) >= 3 * kNumSms) return launch_tc_major<256, 2>(g, st, cls);
    if (g.N % 128 == 0 && base * (g.N / 128) >= 2 * kNumSms) return launch_tc_major<128, 3>(g, st, cls);
    return launch_tc_major<64, 4>(g, st, cls);
  }
  SimtArgs p;
  p.M = g.M; p.N = g.N; p.K = g.K; p.splits = g.splits;
  p.A = static_cast<const float*>(g.A.base); p.lda = g.A.ld; p.a_zrow = g.A.zrow; p.a_zcol = g.A.zcol; p.a_mn = g.a_mn;
  p.B = static_cast<const float*>(g.B.base); p.ldb = g.B.ld; p.b_zrow = g.B.zrow; p.b_zcol = g.B.zcol; p.b_mn = g.b_mn;
  p.epi = g.epi;
  dim3 grid((g.N + 63) / 64, (g.M + 63) / 64, g.batch * g.splits);
  LaunchScope ls(cls, st);
  if (launch_pdl(gemm_f32_simt, grid, dim3(256), 0, st, p) != cudaSuccess) return POETX_ERR_CUDA;
  return last_launch();
}

// -------------------------------------------------------------------- elementwise launches
int ew_grid(long n) { return (int)std::min<long>((n + 255) / 256, (long)kNumSms * 16); }

poetx_status permute_cols(int dt, const void* in, long ld_in, void* out, long ld_out, long rows, int cols,
                          const int32_t* colmap, const int32_t* rowmap, bool scatter, cudaStream_t st) {
  if (rows <= 0) return POETX_OK;
  if (cols > 65536) return POETX_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(colmap)) return POETX_ERR_ALIGNMENT;
  if (dt == BF16 && aligned16(in) && ld_in % 8 == 0 && cols <= 16384) {
    // Bulk-copy kernel: groups of four rows (two above 8192 columns), two groups per block in
    // flight from the start, as many blocks as fit (two per SM at 4096 columns).
    const bool four = cols <= 8192;
    const size_t smem = four ? permute_bulk_smem_bytes<4>(cols) : permute_bulk_smem_bytes<2>(cols);
    auto k = four ? permute_cols_bulk_kernel<4> : permute_cols_bulk_kernel<2>;
    if (!set_smem(k, smem)) return POETX_ERR_CUDA;
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 256, smem) != cudaSuccess || per_sm < 1)
      return POETX_ERR_CUDA;
    const long groups = (rows + (four ? 4 : 2) - 1) / (four ? 4 : 2);
    const int grid = (int)std::min<long>(groups, (long)kNumSms * per_sm);
    LaunchScope ls(POETX_KC_PERMUTE, st);
    if (launch_pdl(k, dim3(grid), dim3(256), smem, st, static_cast<const uint16_t*>(in), ld_in,
                   static_cast<uint16_t*>(out), ld_out, rows, cols, colmap, rowmap, scatter ? 1 : 0) != cudaSuccess)
      return POETX_ERR_CUDA;
  } else if (dt == BF16) {
    // Groups of four rows (two for very wide rows); as many blocks as fit.
    const bool four = permute_smem_bytes<4>(cols) <= 160 * 1024;
    const size_t smem = four ? permute_smem_bytes<4>(cols) : permute_smem_bytes<2>(cols);
    if (smem > 200 * 1024) return POETX_ERR_UNSUPPORTED_SHAPE;
    const long groups = (rows + (four ? 4 : 2) - 1) / (four ? 4 : 2);
    auto k = four ? permute_cols_bf16_kernel<4> : permute_cols_bf16_kernel<2>;
    if (!set_smem(k, smem)) return POETX_ERR_CUDA;
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 256, smem) != cudaSuccess || per_sm < 1)
      return POETX_ERR_CUDA;
    // Rows of at most 4096 columns are software-pipelined across groups: about two groups per
    // block (at least one block per SM); wider rows: as many blocks as fit.
    const long want = cols <= 4096 ? std::min<long>(groups, std::max<long>(kNumSms, (groups + 1) / 2)) : groups;
    const int grid = (int)std::min<long>(want, (long)kNumSms * per_sm);
    LaunchScope ls(POETX_KC_PERMUTE, st);
    if (launch_pdl(k, dim3(grid), dim3(256), smem, st, static_cast<const uint16_t*>(in), ld_in,
                   static_cast<uint16_t*>(out), ld_out, rows, cols, colmap, rowmap, scatter ? 1 : 0) != cudaSuccess)
      return POETX_ERR_CUDA;
  } else {
    const size_t smem = (size_t)cols * 4;
    if (smem > 200 * 1024) return POETX_ERR_UNSUPPORTED_SHAPE;
    auto k = permute_cols_f32_kernel;
    if (!set_smem(k, smem)) return POETX_ERR_CUDA;
    const int grid = (int)std::min<long>(rows, (long)kNumSms * 4);
    LaunchScope ls(POETX_KC_PERMUTE, st);
    k<<<grid, 256, smem, st>>>(static_cast<const float*>(in), ld_in, static_cast<float*>(out), ld_out, rows, cols,
                               colmap, rowmap, scatter ? 1 : 0);
  }
  return last_launch();
}

poetx_status unpack(const float* theta, long nblocks, int b, void* o1, int dt1, long ld1, void* o2, int dt2,
                    long ld2, float* of32, bool add_identity, cudaStream_t st) {
  const long total = nblocks * (long)b * b;
  if (total == 0) return POETX_OK;
  LaunchScope ls(POETX_KC_ELEMENTWISE, st);
  unpack_skew_kernel<<<ew_grid(total), 256, 0, st>>>(theta, nblocks, b, o1, dt1, ld1, o2, dt2, ld2, of32,
                                                      add_identity ? 1 : 0);
  return last_launch();
}

poetx_status pack(const float* GS, long nblocks, int b, float* g, cudaStream_t st) {
  const long total = nblocks * (long)b * b;
  if (total == 0) return POETX_OK;
  LaunchScope ls(POETX_KC_ELEMENTWISE, st);
  pack_antisym_kernel<<<ew_grid(total), 256, 0, st>>>(GS, nblocks, b, g);
  return last_launch();
}

poetx_status reduce_splits(const float* part, int splits, long rows, int cols, float* out, void* out2, int dt2,
                           long ld2, cudaStream_t st) {
  const long total = rows * cols;
  if (total == 0) return POETX_OK;
  LaunchScope ls(POETX_KC_ELEMENTWISE, st);
  reduce_splits_kernel<<<ew_grid(total), 256, 0, st>>>(part, splits, total, rows, cols, out, out2, dt2, ld2);
  return last_launch();
}

// -------------------------------------------------------------------- GEMM building blocks

// W0' GEMM fused with the following block-diagonal factor (b = 256 only): out2 = D . Q^T
// (q_mn = false, forward BD_R) or D . Q (q_mn = true, adjoint of BD_P), D also stored to d1.
bool bd_fusable(int dt, int b, const GemmDesc& g) {
  return dt == BF16 && b == 256 && !g.a_mn && g.N % 256 == 0 && g.batch == 1 && g.splits == 1 && g.K > 0;
}

template <bool BMN, bool QMN>
poetx_status launch_bd_fused(const GemmDesc& g, const void* Q, long q_rows, void* out2, long ld2, cudaStream_t st,
                             int cls) {
  static bool attr_done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return POETX_ERR_CUDA;
  constexpr size_t smem = tc_smem_bytes<256, 4>();
  auto kern = gemm_bd_fused_tc<BMN, QMN>;
  if (!attr_done[dev]) {
    if (!set_smem(kern, smem)) return POETX_ERR_CUDA;
    attr_done[dev] = true;
  }
  CUtensorMap ta, tb, tq;
  if (!make_tmap(&ta, g.A, 64, TC_BM)) return POETX_ERR_CUDA;
  if (!make_tmap(&tb, g.B, 64, BMN ? 64 : 256)) return POETX_ERR_CUDA;
  if (!make_tmap(&tq, view(Q, q_rows, 256, 256), 64, QMN ? 64 : 256)) return POETX_ERR_CUDA;
  FuseArgs a;
  a.M = g.M; a.N = g.N; a.K = g.K;
  a.d1 = g.epi.d1; a.ld1 = g.epi.ld1;
  a.out2 = out2; a.ld2 = ld2;
  dim3 grid(g.N / 256, (g.M + TC_BM - 1) / TC_BM, 1);
  LaunchScope ls(cls, st);
  if (launch_pdl(kern, grid, dim3(128), smem, st, ta, tb, tq, a) != cudaSuccess) return POETX_ERR_CUDA;
  return last_launch();
}

poetx_status run_gemm_bd_fused(const GemmDesc& g, const void* Q, long q_rows, bool q_mn, void* out2, long ld2,
                               cudaStream_t st, int cls) {
  POETX_TRY(check_gemm(g, BF16));
  if (q_rows < g.N || !aligned16(Q) || !aligned16(out2) || ld2 % 8) return POETX_ERR_ALIGNMENT;
  const Epilogue& e = g.epi;
  if (e.d1 && (e.d1_dtype != BF16 || e.alpha1 != 1.f || e.c || e.d2 || e.diag1 || e.split_stride1)) return POETX_ERR_INVALID_ARG;
  if (!g.b_mn && !q_mn) return launch_bd_fused<false, false>(g, Q, q_rows, out2, ld2, st, cls);
  if (!g.b_mn && q_mn) return launch_bd_fused<false, true>(g, Q, q_rows, out2, ld2, st, cls);
  if (g.b_mn && !q_mn) return launch_bd_fused<true, false>(g, Q, q_rows, out2, ld2, st, cls);
  return launch_bd_fused<true, true>(g, Q, q_rows, out2, ld2, st, cls);
}

// 256 x 256 tiles (gemm_w256_tc) for the W0' GEMM when they still occupy three quarters of the
// SMs: plain bf16 store of D, optionally followed by the block factor (b = 256).
bool w256_ok(int dt, const GemmDesc& g) {
  const Epilogue& e = g.epi;
  const bool plain_epi = e.d1 != nullptr && e.d1_dtype == BF16 && e.alpha1 == 1.f && e.beta1 == 0.f && !e.c &&
                         !e.d2 && !e.diag1 && !e.split_stride1;
  return dt == BF16 && !g.a_mn && g.N % 256 == 0 && g.batch == 1 && g.splits == 1 && g.K > 0 && plain_epi &&
         4L * ((g.M + TCW_BM - 1) / TCW_BM) * (g.N / TCW_BN) >= 3L * kNumSms;
}

template <bool BMN, bool QMN, bool Q8 = false>
poetx_status launch_w256(const GemmDesc& g, const void* Q, long q_rows, void* out2, long ld2, cudaStream_t st,
                         int cls) {
  static bool attr_done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return POETX_ERR_CUDA;
  constexpr size_t smem = tcw_smem_bytes();
  auto kern = gemm_w256_tc<BMN, QMN, Q8>;
  if (!attr_done[dev]) {
    if (!set_smem(kern, smem)) return POETX_ERR_CUDA;
    attr_done[dev] = true;
  }
  CUtensorMap ta, tb, tq, td, to;
  if (!make_tmap(&ta, g.A, 64, TCW_BM)) return POETX_ERR_CUDA;
  if (Q8) {
    // int8 codes: a 64 (k) x 256 (n) box of the K-major array, or 256 (n) x 64 (k) of the MN-major one.
    if (!make_tmap(&tb, g.B, BMN ? TCW_BN : 64, BMN ? 64 : TCW_BN, U8)) return POETX_ERR_CUDA;
  } else if (!make_tmap(&tb, g.B, 64, BMN ? 64 : TCW_BN)) {
    return POETX_ERR_CUDA;
  }
  // Store boxes of D: 64 columns x 128 rows (one half's K chunk).
  if (!make_tmap(&td, view(g.epi.d1, g.M, g.N, g.epi.ld1), 64, TC_BM)) return POETX_ERR_CUDA;
  if (out2 != nullptr) {
    if (!make_tmap(&tq, view(Q, q_rows, 256, 256), 64, QMN ? 64 : 256)) return POETX_ERR_CUDA;
    // Store boxes of the block-factor result: 64 columns x 32 rows (one warp's rows).
    if (!make_tmap(&to, view(out2, g.M, g.N, ld2), 64, 32)) return POETX_ERR_CUDA;
  } else {
    tq = ta;  // unused without the block factor
    to = ta;
  }
  WideArgs a = {};
  a.M = g.M; a.N = g.N; a.K = g.K;
  a.d1 = g.epi.d1; a.ld1 = g.epi.ld1;
  a.out2 = out2; a.ld2 = ld2;
  a.bscale = g.b_scale;
  a.b_early = g.b_static ? 1 : 0;
  dim3 grid(g.N / TCW_BN, (g.M + TCW_BM - 1) / TCW_BM, 1);
  LaunchScope ls(cls, st);
  if (launch_pdl_prio(kern, grid, dim3(tcw_threads(Q8)), smem, st, true, ta, tb, tq, td, to, a) != cudaSuccess)
    return POETX_ERR_CUDA;
  return last_launch();
}

// POET-XQ W0' GEMM: B is int8 codes with per-row scales (g.b_scale), dequantised in the kernel.
// Always the 256 x 256 kernel (its converter warps are the only dequantising path): N in whole
// 256-column tiles, rows of codes 16-byte aligned.
poetx_status run_w_gemm_q8(const GemmDesc& g, const void* Q, long q_rows, bool q_mn, void* out2, long ld2,
                           cudaStream_t st, int cls) {
  const Epilogue& e = g.epi;
  if (g.M <= 0 || g.K <= 0 || g.a_mn || g.batch != 1 || g.splits != 1 || g.N % TCW_BN) return POETX_ERR_UNSUPPORTED_SHAPE;
  if (!e.d1 || e.d1_dtype != BF16 || e.alpha1 != 1.f || e.beta1 != 0.f || e.c || e.d2 || e.diag1 || e.split_stride1)
    return POETX_ERR_INVALID_ARG;
  if (!view_fits(g.A, false, g.M, g.K, 1) || !view_fits(g.B, g.b_mn, g.N, g.K, 1)) return POETX_ERR_INVALID_ARG;
  if (!aligned16(g.A.base) || g.A.ld % 8 || !aligned16(g.B.base) || g.B.ld % 16 || !aligned16(e.d1) || e.ld1 % 8 ||
      !aligned16(g.b_scale))
    return POETX_ERR_ALIGNMENT;
  if (out2 == nullptr) {
    return g.b_mn ? launch_w256<true, false, true>(g, nullptr, 0, nullptr, 0, st, cls)
                  : launch_w256<false, false, true>(g, nullptr, 0, nullptr, 0, st, cls);
  }
  if (q_rows < g.N || !aligned16(Q) || !aligned16(out2) || ld2 % 8) return POETX_ERR_ALIGNMENT;
  if (!g.b_mn && !q_mn) return launch_w256<false, false, true>(g, Q, q_rows, out2, ld2, st, cls);
  if (!g.b_mn && q_mn) return launch_w256<false, true, true>(g, Q, q_rows, out2, ld2, st, cls);
  if (g.b_mn && !q_mn) return launch_w256<true, false, true>(g, Q, q_rows, out2, ld2, st, cls);
  return launch_w256<true, true, true>(g, Q, q_rows, out2, ld2, st, cls);
}

// The W0' GEMM D = A . B^T -> d1, and (out2 != null, b = 256) out2 = D . Q^T or D . Q.
poetx_status run_w_gemm(int dt, const GemmDesc& g, const void* Q, long q_rows, bool q_mn, void* out2, long ld2,
                        cudaStream_t st, int cls = POETX_KC_W_GEMM) {
  if (g.b_scale != nullptr) return dt == BF16 ? run_w_gemm_q8(g, Q, q_rows, q_mn, out2, ld2, st, cls) : POETX_ERR_INVALID_ARG;
  if (out2 == nullptr) {
    if (!w256_ok(dt, g)) return run_gemm(dt, g, st, cls);
    POETX_TRY(check_gemm(g, BF16));
    return g.b_mn ? launch_w256<true, false>(g, nullptr, 0, nullptr, 0, st, cls)
                  : launch_w256<false, false>(g, nullptr, 0, nullptr, 0, st, cls);
  }
  if (!w256_ok(dt, g)) return run_gemm_bd_fused(g, Q, q_rows, q_mn, out2, ld2, st, cls);
  POETX_TRY(check_gemm(g, BF16));
  if (q_rows < g.N || !aligned16(Q) || !aligned16(out2) || ld2 % 8) return POETX_ERR_ALIGNMENT;
  if (!g.b_mn && !q_mn) return launch_w256<false, false>(g, Q, q_rows, out2, ld2, st, cls);
  if (!g.b_mn && q_mn) return launch_w256<false, true>(g, Q, q_rows, out2, ld2, st, cls);
  if (g.b_mn && !q_mn) return launch_w256<true, false>(g, Q, q_rows, out2, ld2, st, cls);
  return launch_w256<true, true>(g, Q, q_rows, out2, ld2, st, cls);
}

// Out[:, blk z] = In[:, blk z] . Q_z^T  (forward block-diagonal application; tokens are rows).
poetx_status bd_forward(int dt, long n, int d, int b, const void* in, const void* Q, void* out, cudaStream_t st) {
  GemmDesc g;
  g.M = (int)n; g.N = b; g.K = b; g.batch = d / b;
  g.A = view(in, n, d, d, 0, b);
  g.B = view(Q, d, b, b, b, 0);
  g.epi.d1 = out; g.epi.d1_dtype = dt; g.epi.ld1 = d; g.epi.zcol1 = b;
  return run_gemm(dt, g, st, POETX_KC_BD_GEMM);
}

// Out[:, blk z] = In[:, blk z] . Q_z  (adjoint of bd_forward w.r.t. its input).
poetx_status bd_backward(int dt, long n, int d, int b, const void* in, const void* Q, void* out, cudaStream_t st,
                         bool q_static = false) {
  GemmDesc g;
  g.b_static = q_static;
  g.M = (int)n; g.N = b; g.K = b; g.batch = d / b;
  g.A = view(in, n, d, d, 0, b);
  g.B = view(Q, d, b, b, b, 0);
  g.b_mn = true;
  g.epi.d1 = out; g.epi.d1_dtype = dt; g.epi.ld1 = d; g.epi.zcol1 = b;
  return run_gemm(dt, g, st, POETX_KC_BD_GEMM);
}

// Gpart[s][z] = Lhs[:, blk z]^T . Rhs[:, blk z] over split s of the tokens (f32 partials).
// Split-K factor of the block-gradient GEMMs: enough CTAs of 128 x 128 tiles (bf16) to fill the
// SMs (each operand panel is then fetched by two CTAs instead of four with 128 x 64 tiles), no
// split when the tiles alone do.
int grad_splits(int dt, long n, int nb, int b) {
  const long tiles = dt == BF16 ? (long)nb * ((b + 127) / 128) * ((b + 127) / 128)
                                : (long)nb * ((b + 63) / 64) * ((b + 63) / 64);
  const long kt = dt == BF16 ? (n + 63) / 64 : (n + 15) / 16;
  long s = std::max<long>(1, kNumSms / std::max<long>(1, tiles));
  s = std::min<long>(s, std::max<long>(1, kt / 4));
  return (int)std::max<long>(1, std::min<long>(s, 64));
}

// reduce: every split adds its partial into the one [nb*b, b] tile set at `part` (zeroed by the
// caller) instead of writing its own.
poetx_status block_grads(int dt, long n, int d, int b, const void* lhs, const void* rhs, float* part, int splits,
                         cudaStream_t st, bool few_ctas = false, bool rhs_static = false, bool reduce = false) {
  GemmDesc g;
  g.b_static = rhs_static;
  g.M = b; g.N = b; g.K = (int)n; g.batch = d / b; g.splits = splits;
  g.A = view(lhs, n, d, d, 0, b); g.a_mn = true;
  g.B = view(rhs, n, d, d, 0, b); g.b_mn = true;
  g.epi.d1 = part; g.epi.d1_dtype = F32; g.epi.ld1 = b; g.epi.zrow1 = b;
  g.epi.split_stride1 = reduce ? 0 : (long)d * b;
  g.epi.red1 = reduce ? 1 : 0;
  // few_ctas: the widest tile and the deep ring whatever the CTA count, for a launch that runs
  // beside a GEMM on the SMs that one leaves free.
  if (few_ctas && dt == BF16 && b % 256 == 0) {
    POETX_TRY(check_gemm(g, dt));
    return launch_tc_major<256, 4>(g, st, POETX_KC_GRAD_GEMM);
  }
  return run_gemm(dt, g, st, POETX_KC_GRAD_GEMM);
}

// ------------------------------------------------------------------------- CNP forward
size_t cnp_fwd_generic_ws(int b, int k, int dt, long nb) {
  if (k == 0 || nb == 0) return 0;
  const size_t blk = (size_t)nb * b * b;
  Plan p;
  p.take(blk * 4);                  // S (f32)
  if (dt == BF16) p.take(blk * 2);  // S (bf16 operand)
  if (k >= 2) {
    p.take(blk * esize(dt));        // M_j ping-pong
    p.take(blk * esize(dt));
    p.take(blk * 4);                // T = S + M_k (f32)
  }
  return p.total;
}

// Q = (I + S)(I + S + ... + S^k) by the Horner recursion N_1 = I + S, N_j = I + S.N_{j-1},
// Q = N_k + S.N_k, carried on M_j = N_j - I (small, so bf16 intermediates stay accurate):
//   M_1 = S;  M_j = S + S.M_{j-1};  Q = I + (S + M_k) + S.M_k.
// The product that yields M_k also writes T = S + M_k = 2S + S.M_{k-1} in fp32, and the exact
// I + T part of Q is added in fp32 in the last epilogue (replication review, "Summary": the
// fused CNP reuses the lower powers across terms).
poetx_status cnp_fwd_generic(int b, int k, int dt, long nb, const float* theta, void* Q, char* ws, cudaStream_t st) {
  if (nb == 0) return POETX_OK;
  if (k == 0) return unpack(theta, nb, b, Q, dt, b, nullptr, dt, 0, nullptr, true, st);
  const size_t blk = (size_t)nb * b * b;
  Plan p;
  float* S32 = reinterpret_cast<float*>(ws + p.take(blk * 4));
  void* Sop = dt == BF16 ? static_cast<void*>(ws + p.take(blk * 2)) : static_cast<void*>(S32);
  void* Mbuf[2] = {nullptr, nullptr};
  float* T32 = nullptr;
  if (k >= 2) {
    Mbuf[0] = ws + p.take(blk * esize(dt));
    Mbuf[1] = ws + p.take(blk * esize(dt));
    T32 = reinterpret_cast<float*>(ws + p.take(blk * 4));
  }
  POETX_TRY(unpack(theta, nb, b, dt == BF16 ? Sop : nullptr, dt, b, nullptr, dt, 0, S32, false, st));
  auto chain = [&](const void* Mprev) {
    GemmDesc g;
    g.M = b; g.N = b; g.K = b; g.batch = (int)nb;
    g.A = view(Sop, nb * b, b, b, b, 0);
    g.B = view(Mprev, nb * b, b, b, b, 0); g.b_mn = true;
    g.epi.d1_dtype = dt; g.epi.ld1 = b; g.epi.zrow1 = b;
    g.epi.c_dtype = F32; g.epi.ldc = b; g.epi.zrowc = b;
    return g;
  };
  const void* Mprev = Sop;  // M_1 = S
  for (int j = 2; j <= k; ++j) {
    GemmDesc g = chain(Mprev);
    g.epi.d1 = Mbuf[j & 1];
    g.epi.alpha1 = 1.f; g.epi.beta1 = 1.f; g.epi.c = S32;   // M_j = S.M_{j-1} + S
    if (j == k) {                                            // T = S + M_k = S.M_{k-1} + 2S
      g.epi.d2 = T32; g.epi.ld2 = b; g.epi.zrow2 = b; g.epi.alpha2 = 1.f; g.epi.beta2 = 2.f;
    }
    POETX_TRY(run_gemm(dt, g, st, POETX_KC_CNP_GEMM));
    Mprev = Mbuf[j & 1];
  }
  GemmDesc g = chain(Mprev);                                 // Q = I + T + S.M_k
  g.epi.d1 = Q; g.epi.alpha1 = 1.f; g.epi.diag1 = 1;
  if (k == 1) { g.epi.c = S32; g.epi.beta1 = 2.f; }          // T = S + M_1 = 2S
  else { g.epi.c = T32; g.epi.beta1 = 1.f; }
  return run_gemm(dt, g, st, POETX_KC_CNP_GEMM);
}

// ------------------------------------------------------------------------- CNP backward
size_t cnp_bwd_generic_ws(int b, int k, int dt, long nb) {
  if (nb == 0) return 0;
  const size_t blk = (size_t)nb * b * b;
  Plan p;
  p.take(blk * 4);  // G (f32)
  if (k >= 1) {
    p.take(blk * 4);                               // E (f32), then G_S
    p.take(blk * 4);                               // S (f32)
    if (dt == BF16) p.take(blk * 2);               // S (bf16 operand)
    p.take(blk * (size_t)k * esize(dt));           // A-stack [G | Gbar_k | ... | Gbar_2]
    p.take(blk * (size_t)k * esize(dt));           // B-stack [M_k | ... | M_1]
  }
  return p.total;
}

// Packed gradient from G = dL/dQ (split-K partials) by the adjoint of the Horner recursion
// N_0 = I, N_j = I + S.N_{j-1}, Q = (I + S).N_k:
//   G_S = G.N_k^T + sum_{j=1..k} Gbar_j.N_{j-1}^T,  Gbar_k = (I + S^T).G,  Gbar_{j-1} = S^T.Gbar_j,
// then g[p(i,j)] = G_S[i][j] - G_S[j][i].  With N_j = I + M_j and S^T = -S this is
//   G_S = E + [G | Gbar_k | ... | Gbar_2] . [M_k | ... | M_1]^T,   E = G + sum_{j=1..k} Gbar_j,
// one long-K product plus an fp32 running sum E (the dominant 2G term never rounds to bf16).
poetx_status cnp_bwd_generic(int b, int k, int dt, long nb, const float* theta, const float* part, int splits,
                             float* grad, char* ws, cudaStream_t st) {
  if (nb == 0) return POETX_OK;
  const size_t blk = (size_t)nb * b * b;
  const long rows = nb * b;
  Plan p;
  float* G32 = reinterpret_cast<float*>(ws + p.take(blk * 4));
  if (k == 0) {
    POETX_TRY(reduce_splits(part, splits, rows, b, G32, nullptr, F32, 0, st));
    return pack(G32, nb, b, grad, st);
  }
  float* E = reinterpret_cast<float*>(ws + p.take(blk * 4));
  float* S32 = reinterpret_cast<float*>(ws + p.take(blk * 4));
  void* Sop = dt == BF16 ? static_cast<void*>(ws + p.take(blk * 2)) : static_cast<void*>(S32);
  char* Ast = ws + p.take(blk * (size_t)k * esize(dt));
  char* Bst = ws + p.take(blk * (size_t)k * esize(dt));
  const long kb = (long)k * b;
  const int es = esize(dt);
  auto aslot = [&](int t) { return static_cast<void*>(Ast + (size_t)t * b * es); };
  auto bslot = [&](int t) { return static_cast<void*>(Bst + (size_t)t * b * es); };

  POETX_TRY(reduce_splits(part, splits, rows, b, G32, aslot(0), dt, kb, st));
  POETX_TRY(unpack(theta, nb, b, dt == BF16 ? Sop : nullptr, dt, b, bslot(k - 1), dt, kb, S32, false, st));

  auto chain_gemm = [&](const void* Bsrc) {
    GemmDesc g;
    g.M = b; g.N = b; g.K = b; g.batch = (int)nb;
    g.A = view(Sop, rows, b, b, b, 0);
    g.B = view(Bsrc, rows, b, kb, b, 0); g.b_mn = true;
    return g;
  };
  // M_j = S + S.M_{j-1} into B-slot k-j.
  for (int j = 2; j <= k; ++j) {
    GemmDesc g = chain_gemm(bslot(k - j + 1));
    g.epi.d1 = bslot(k - j); g.epi.d1_dtype = dt; g.epi.ld1 = kb; g.epi.zrow1 = b;
    g.epi.alpha1 = 1.f; g.epi.beta1 = 1.f;
    g.epi.c = S32; g.epi.c_dtype = F32; g.epi.ldc = b; g.epi.zrowc = b;
    POETX_TRY(run_gemm(dt, g, st, POETX_KC_CNP_ADJ));
  }
  // Gbar_k = G - S.G into A-slot 1 (k >= 2);  E = 2G - S.G.
  {
    GemmDesc g = chain_gemm(aslot(0));
    if (k >= 2) {
      g.epi.d1 = aslot(1); g.epi.d1_dtype = dt; g.epi.ld1 = kb; g.epi.zrow1 = b;
      g.epi.alpha1 = -1.f; g.epi.beta1 = 1.f;
    }
    g.epi.c = G32; g.epi.c_dtype = F32; g.epi.ldc = b; g.epi.zrowc = b;
    g.epi.d2 = E; g.epi.ld2 = b; g.epi.zrow2 = b; g.epi.alpha2 = -1.f; g.epi.beta2 = 2.f; g.epi.accum2 = 0;
    POETX_TRY(run_gemm(dt, g, st, POETX_KC_CNP_ADJ));
  }
  // Gbar_j = -S.Gbar_{j+1} (Gbar_{j+1} in A-slot k-j) into A-slot k-j+1 (j >= 2);  E += Gbar_j.
  for (int j = k - 1; j >= 1; --j) {
    GemmDesc g = chain_gemm(aslot(k - j));
    if (j >= 2) {
      g.epi.d1 = aslot(k - j + 1); g.epi.d1_dtype = dt; g.epi.ld1 = kb; g.epi.zrow1 = b;
      g.epi.alpha1 = -1.f; g.epi.beta1 = 0.f;
    }
    g.epi.d2 = E; g.epi.ld2 = b; g.epi.zrow2 = b; g.epi.alpha2 = -1.f; g.epi.beta2 = 0.f; g.epi.accum2 = 1;
    POETX_TRY(run_gemm(dt, g, st, POETX_KC_CNP_ADJ));
  }
  // G_S = E + A-stack . B-stack^T  (K = k.b), written over E.
  {
    GemmDesc g;
    g.M = b; g.N = b; g.K = (int)kb; g.batch = (int)nb;
    g.A = view(Ast, rows, kb, kb, b, 0);
    g.B = view(Bst, rows, kb, kb, b, 0);
    g.epi.d1 = E; g.epi.d1_dtype = F32; g.epi.ld1 = b; g.epi.zrow1 = b; g.epi.alpha1 = 1.f; g.epi.beta1 = 1.f;
    g.epi.c = E; g.epi.c_dtype = F32; g.epi.ldc = b; g.epi.zrowc = b;
    POETX_TRY(run_gemm(dt, g, st, POETX_KC_CNP_ADJ));
  }
  return pack(E, nb, b, grad, st);
}

// ----------------------------------------------------------------- on-chip CNP (bf16 path)
// One launch runs the whole CNP forward (or adjoint) of up to two block sets (the R and P sides
// of a layer) with every operand on chip; see cnp_onchip.cuh.  Used for bf16 and b <= 256; it
// needs no global scratch.
bool cnp_fused_ok(int b, int dt) { return dt == BF16 && (b == 64 || b == 128 || b == 256); }

size_t cnp_fwd_fused_ws(int, int, long) { return 0; }
size_t cnp_bwd_fused_ws(int, int, long) { return 0; }

struct CnpSide {
  long nb = 0;
  const float* theta = nullptr;
  void* Q = nullptr;                // forward output
  const float* part = nullptr;      // adjoint: split-K partials of G
  int splits = 1;
  float* grad = nullptr;            // adjoint output
};

template <int B, bool ADJ>
poetx_status launch_cnp_chip(int k, const CnpSide* sides, int nsides, cudaStream_t st,
                             const CnpGather* gather = nullptr) {
  using C = ChipCfg<B>;
  static bool attr_done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return POETX_ERR_CUDA;
  auto kern = cnp_chip_kernel<B, ADJ>;
  if (!attr_done[dev]) {
    if (!set_smem(kern, C::SMEM)) return POETX_ERR_CUDA;
    attr_done[dev] = true;
  }
  CnpChipArgs a;
  std::memset(&a, 0, sizeof(a));
  a.nseg = nsides;
  a.k = k;
  long nb_total = 0;
  for (int q = 0; q < nsides; ++q) {
    const CnpSide& sd = sides[q];
    CnpChipSide& S = a.seg[q];
    S.nb = (int)sd.nb;
    S.theta = sd.theta;
    S.part = sd.part;
    S.splits = sd.splits;
    S.grad = sd.grad;
    nb_total += sd.nb;
    if (!aligned16(sd.theta)) return POETX_ERR_ALIGNMENT;
    if (!ADJ) {
      if (!aligned16(sd.Q)) return POETX_ERR_ALIGNMENT;
      // Q leaves through TMA stores of (64 columns x rows-per-CTA) boxes.
      if (!make_tmap(&S.tmQ, view(sd.Q, sd.nb * B, B, B), 64, C::ROWS)) return POETX_ERR_CUDA;
    } else {
      if (!aligned16(sd.part) || sd.splits < 1) return POETX_ERR_ALIGNMENT;
      // G partials arrive through TMA loads of (32 columns x rows-per-CTA) fp32 boxes.
      if (!make_tmap(&S.tmG, view(sd.part, (long)sd.splits * sd.nb * B, B, B), 32, C::ROWS, F32))
        return POETX_ERR_CUDA;
    }
  }
  if (nb_total == 0) return POETX_OK;
  if (nb_total * C::NCTA > 0x7fffffffL - 1024) return POETX_ERR_UNSUPPORTED_SHAPE;
  a.ncnp = (int)(nb_total * C::NCTA);
  if (gather != nullptr) a.gather = *gather;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.ncnp + a.gather.nblk), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (C::PAIR) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  LaunchScope ls(ADJ ? POETX_KC_CNP_ADJ : POETX_KC_CNP_GEMM, st);
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return POETX_ERR_CUDA;
  return last_launch();
}

// SMs of the current device (cached per device).
int device_sms() {
  static int sms[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return kNumSms;
  if (sms[dev] == 0 && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms[dev] = kNumSms;
  return sms[dev];
}

// CNP (forward or adjoint) of both sides of a b = 256 layer (one SM pair per block) with a bf16
// column permutation on the SMs the pairs leave free, in the same launch: the forward's input
// gather U = X[:, pi_R], the adjoint's scatter dX[:, pi_R] = dU.  Returns false (nothing
// launched) where that does not fit: other block sizes, too few free SMs, rows too wide for the
// launch's shared memory.
template <bool ADJ>
bool cnp_with_permute(int b, int k, const CnpSide* sides, int nsides, const void* in, long ld_in, void* out,
                      long ld_out, long rows, int cols, const int32_t* colmap, bool scatter, cudaStream_t st,
                      poetx_status* status) {
  if (b != 256 || rows <= 0) return false;
  long nb_total = 0;
  for (int q = 0; q < nsides; ++q) nb_total += sides[q].nb;
  const long free_sms = (long)device_sms() - 2 * nb_total;
  if (free_sms < 16 || cols > 8192 || cols % 8 ||
      permute_bulk_smem_bytes<4, kSpareSlots>(cols) + 1024 > ChipCfg<256>::SMEM || !aligned16(in) ||
      !aligned16(out) || !aligned16(colmap) || ld_in % 8 || ld_out % 8)
    return false;
  CnpGather g;
  g.in = static_cast<const uint16_t*>(in); g.ld_in = ld_in;
  g.out = static_cast<uint16_t*>(out); g.ld_out = ld_out;
  g.rows = rows; g.cols = cols; g.colmap = colmap; g.scatter = scatter ? 1 : 0;
  const long groups = (rows + 3) / 4;
  g.nblk = (int)std::min<long>(free_sms & ~1L, (groups + 1) & ~1L);  // whole clusters of two
  *status = launch_cnp_chip<256, ADJ>(k, sides, nsides, st, &g);
  return true;
}

template <bool ADJ>
poetx_status run_cnp_chip(int b, int k, const CnpSide* sides, int nsides, cudaStream_t st) {
  if (b == 256) return launch_cnp_chip<256, ADJ>(k, sides, nsides, st);
  if (b == 128) return launch_cnp_chip<128, ADJ>(k, sides, nsides, st);
  if (b == 64) return launch_cnp_chip<64, ADJ>(k, sides, nsides, st);
  return POETX_ERR_UNSUPPORTED_SHAPE;
}

// Forward: Q of every block of the given sides (one launch).
poetx_status cnp_fwd_fused(int b, int k, const CnpSide* sides, int nsides, cudaStream_t st) {
  return run_cnp_chip<false>(b, k, sides, nsides, st);
}
// Adjoint: packed gradients from the split-K partials of G = dL/dQ (one launch).
poetx_status cnp_bwd_fused(int b, int k, const CnpSide* sides, int nsides, cudaStream_t st) {
  return run_cnp_chip<true>(b, k, sides, nsides, st);
}

// Scratch of the CNP forward / adjoint for nb blocks (fused path for bf16 and b <= 256).
size_t cnp_fwd_ws(int b, int k, int dt, long nb) {
  return cnp_fused_ok(b, dt) ? cnp_fwd_fused_ws(b, k, nb) : cnp_fwd_generic_ws(b, k, dt, nb);
}
size_t cnp_bwd_ws(int b, int k, int dt, long nb) {
  return cnp_fused_ok(b, dt) ? cnp_bwd_fused_ws(b, k, nb) : cnp_bwd_generic_ws(b, k, dt, nb);
}

poetx_status cnp_fwd_run(int b, int k, int dt, long nb, const float* theta, void* Q, char* ws, cudaStream_t st) {
  if (!cnp_fused_ok(b, dt)) return cnp_fwd_generic(b, k, dt, nb, theta, Q, ws, st);
  CnpSide sd;
  sd.nb = nb; sd.theta = theta; sd.Q = Q;
  return cnp_fwd_fused(b, k, &sd, 1, st);
}

// ------------------------------------------------------------------------- layer plans
struct FwdPlan {
  size_t U, V, Yp, Z, total;
};
FwdPlan fwd_plan(const poetx_desc* d, long n) {
  const size_t e = esize(d->dtype);
  Plan p;
  FwdPlan f;
  f.U = d->mode == POETX_MEM ? p.take(n * d->d_in * e) : 0;
  f.V = p.take(n * d->d_in * e);
  f.Yp = p.take(n * d->d_out * e);
  f.Z = d->mode == POETX_MEM ? p.take(n * d->d_out * e) : 0;
  f.total = p.total;
  return f;
}

struct BwdPlan {
  size_t dYp, dZ, dV, U, dU, V, Z, GpR, GpP, cnpR, cnpP, total;
  int sR, sP;
};
BwdPlan bwd_plan(const poetx_desc* d, long n) {
  const size_t e = esize(d->dtype);
  const int b = d->b, nbo = d->d_out / b, nbi = d->d_in / b;
  BwdPlan w;
  Plan p;
  w.dYp = p.take(n * d->d_out * e);
  w.dZ = p.take(n * d->d_out * e);
  w.dV = p.take(n * d->d_in * e);
  w.U = d->mode == POETX_MEM ? p.take(n * d->d_in * e) : 0;
  w.dU = p.take(n * d->d_in * e);
  w.V = d->mode == POETX_MEM ? p.take(n * d->d_in * e) : 0;
  w.Z = d->mode == POETX_MEM ? p.take(n * d->d_out * e) : 0;
  w.sR = d->dtype == BF16 && b == 256 ? 1 : grad_splits(d->dtype, n, nbo, b);
  w.sP = grad_splits(d->dtype, n, nbi, b);
  w.GpR = p.take((size_t)w.sR * nbo * b * b * 4);
  w.GpP = p.take((size_t)w.sP * nbi * b * b * 4);
  w.cnpR = p.take(cnp_bwd_ws(b, d->k, d->dtype, nbo));
  w.cnpP = p.take(cnp_bwd_ws(b, d->k, d->dtype, nbi));
  w.total = p.total;
  return w;
}

// Scratch of poetx_cnp: the two sides run concurrently and need disjoint regions.
size_t cnp_layer_ws(const poetx_desc* d) {
  return align256(cnp_fwd_ws(d->b, d->k, d->dtype, d->d_out / d->b)) +
         align256(cnp_fwd_ws(d->b, d->k, d->dtype, d->d_in / d->b));
}

struct MergePlan {
  size_t T, M2, inv, sigL, sigR, total;
};
MergePlan merge_plan(const poetx_desc* d) {
  const size_t e = esize(d->dtype);
  MergePlan m;
  Plan p;
  m.T = p.take((size_t)d->d_out * d->d_in * e);
  m.M2 = p.take((size_t)d->d_out * d->d_in * e);
  m.inv = p.take((size_t)std::max(d->d_in, d->d_out) * 4);
  m.sigL = p.take((size_t)d->d_out * 4);
  m.sigR = p.take((size_t)d->d_in * 4);
  m.total = p.total;
  return m;
}

// Weight-centric comparator (the original POET order): the transformed weight is formed first.
//   forward:  T = W0'.BD_P, M = BD_R.T, W = Pi_L^T M Pi_R (original basis), Y = X.W^T
//   backward: dX = dY.W, dW = dY^T.X, dM = Pi_L dW Pi_R^T, G_R,i = dM[blk i,:].T[blk i,:]^T,
//             B1 = BD_R.W0', G_P,j = B1[:,blk j]^T.dM[:,blk j], then the CNP adjoint.
// The caller keeps `wc_saved` = [W | T] (2 d_out d_in elements) from the forward for the backward.
struct WcPlan {
  size_t M2, invL, invR, dW, dM, B1, GpR, GpP, cnpR, cnpP, total;
};
WcPlan wc_plan(const poetx_desc* d) {
  const size_t e = esize(d->dtype), w = (size_t)d->d_out * d->d_in * e;
  const int b = d->b;
  WcPlan m;
  Plan p;
  m.M2 = p.take(w);
  m.invL = p.take((size_t)d->d_out * 4);
  m.invR = p.take((size_t)d->d_in * 4);
  m.dW = p.take(w);
  m.dM = p.take(w);
  m.B1 = p.take(w);
  m.GpR = p.take((size_t)d->d_out * b * 4);
  m.GpP = p.take((size_t)d->d_in * b * 4);
  m.cnpR = p.take(cnp_bwd_ws(b, d->k, d->dtype, d->d_out / b));
  m.cnpP = p.take(cnp_bwd_ws(b, d->k, d->dtype, d->d_in / b));
  m.total = p.total;
  return m;
}

// Every value in [0, n) exactly once.
bool is_bijection(const int32_t* p, int n) {
  std::vector<unsigned char> seen((size_t)std::max(n, 0), 0);
  for (int i = 0; i < n; ++i) {
    const int32_t v = p[i];
    if (v < 0 || v >= n || seen[v]) return false;
    seen[v] = 1;
  }
  return true;
}

// With POETX_DEBUG set (and not "0") in the environment, read once per process, the entry points
// that take permutations copy them to the host in stream order and check that they are
// bijections before anything is launched.  Skipped while the stream is being captured, where a
// synchronising copy is not allowed.
bool debug_checks() {
  static const bool on = [] {
    const char* e = std::getenv("POETX_DEBUG");
    return e != nullptr && *e != 0 && std::strcmp(e, "0") != 0;
  }();
  return on;
}

poetx_status debug_check_perms(cudaStream_t st, std::initializer_list<std::pair<const int32_t*, int>> perms) {
  if (!debug_checks()) return POETX_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return POETX_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return POETX_OK;
  for (const auto& pr : perms) {
    std::vector<int32_t> h((size_t)std::max(pr.second, 0));
    if (pr.second > 0 &&
        cudaMemcpyAsync(h.data(), pr.first, (size_t)pr.second * 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return POETX_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return POETX_ERR_CUDA;
    if (!is_bijection(h.data(), pr.second)) return POETX_ERR_INVALID_ARG;
  }
  return POETX_OK;
}

poetx_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (p == nullptr) return POETX_ERR_INVALID_ARG;
    if (!aligned16(p)) return POETX_ERR_ALIGNMENT;
  }
  return POETX_OK;
}

poetx_status check_ws(const void* ws, size_t have, size_t need) {
  if (need == 0) return POETX_OK;
  if (ws == nullptr || have < need) return POETX_ERR_WORKSPACE;
  if (!aligned16(ws)) return POETX_ERR_ALIGNMENT;
  return POETX_OK;
}

// Forward chain into caller buffers; `Z` receives the W0'-GEMM output.
poetx_status forward_chain(const poetx_desc* d, long n, const void* X, const void* W0p, const float* W0s,
                           const int32_t* pL, const int32_t* pR, const void* QR, const void* QP, void* Y, void* Z,
                           char* U, char* V, char* Yp, cudaStream_t st, bool gathered = false) {
  const int dt = d->dtype, b = d->b;
  if (!gathered) POETX_TRY(permute_cols(dt, X, d->d_in, U, d->d_in, n, d->d_in, pR, nullptr, false, st));
  POETX_TRY(bd_forward(dt, n, d->d_in, b, U, QP, V, st));
  GemmDesc g;
  g.M = (int)n; g.N = d->d_out; g.K = d->d_in;
  g.A = view(V, n, d->d_in, d->d_in);
  g.B = view(W0p, d->d_out, d->d_in, d->d_in);
  g.b_scale = W0s;  // POET-XQ: W0' is int8 codes with per-row scales
  g.b_static = true;  // W0' is the caller's, not the output of the launch before (BD_P)
  g.epi.d1 = Z; g.epi.d1_dtype = dt; g.epi.ld1 = d->d_out;
  if (Y == nullptr) return run_w_gemm(dt, g, nullptr, 0, false, nullptr, 0, st);  // recompute only (mem-mode backward)
  if (bd_fusable(dt, b, g)) {
    // Z = V.W0'^T and Y'_i = Z_i.Q_R,i^T in one kernel.
    POETX_TRY(run_w_gemm(dt, g, QR, d->d_out, false, Yp, d->d_out, st));
  } else {
    POETX_TRY(run_w_gemm(dt, g, nullptr, 0, false, nullptr, 0, st));
    POETX_TRY(bd_forward(dt, n, d->d_out, b, Z, QR, Yp, st));
  }
  return permute_cols(dt, Yp, d->d_out, Y, d->d_out, n, d->d_out, pL, nullptr, true, st);
}

// ------------------------------------------------------------ allocation-free CNP forward
// Built-in scratch for poetx_cnp_blocks_noalloc.  Some callers cannot hand the library a
// workspace: a plugin living inside a host framework that owns every device allocation and
// exposes no allocator to it, or a latency-critical loop that must never pay for cudaMalloc
// (which can synchronise the device).  For them the CNP forward runs out of this fixed array,
// which every GPU that loads the library keeps until the process exits.  All calls on a device
// share it, so calls that overlap in time on the GPU (different streams, no ordering) race on
// it.  Nothing in it has to start at zero: the CNP forward writes every scratch element it
// reads in the same call.
constexpr size_t kNoAllocScratchBytes = POETX_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_cnp_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the built-in scratch on the current device.  In host code the array's
// name is only a host-side stand-in; the real address comes from cudaGetSymbolAddress, looked
// up once per device (with that device current) and cached.
poetx_status noalloc_scratch(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return POETX_ERR_CUDA;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_cnp_noalloc_scratch) != cudaSuccess || p == nullptr) return POETX_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = static_cast<char*>(g_noalloc_addr[dev]);
  return POETX_OK;
}

}  // namespace

// =============================================================================== C ABI
extern "C" {

poetx_status poetx_adamw_step(const poetx_adamw_cfg* cfg, long long n, int t, float* theta, const float* grad,
                              float* m, float* v, poetx_stream stream) {
  if (cfg == nullptr || n < 0 || t < 1) return POETX_ERR_INVALID_ARG;
  if (!(cfg->lr >= 0.f) || !(cfg->gamma >= 0.f) || !(cfg->beta1 >= 0.f && cfg->beta1 < 1.f) ||
      !(cfg->beta2 >= 0.f && cfg->beta2 < 1.f) || !(cfg->eps > 0.f) || !(cfg->weight_decay >= 0.f))
    return POETX_ERR_INVALID_ARG;
  if (n == 0) return POETX_OK;
  POETX_TRY(check_ptrs({theta, grad, m, v}));
  const double bc1 = 1.0 - std::pow((double)cfg->beta1, (double)t);
  const double bc2 = 1.0 - std::pow((double)cfg->beta2, (double)t);
  AdamwArgs a;
  a.eta = cfg->gamma * cfg->lr;
  a.beta1 = cfg->beta1; a.beta2 = cfg->beta2;
  a.inv_bc1 = (float)(1.0 / bc1);
  a.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  a.eps = cfg->eps; a.decay = cfg->weight_decay;
  const long n4 = (long)(n / 4);
  const int grid = (int)std::max<long>(1, std::min<long>((n4 + 255) / 256, (long)kNumSms * 8));
  LaunchScope ls(POETX_KC_OPTIMIZER, stream);
  if (launch_pdl(adamw_kernel, dim3(grid), dim3(256), 0, stream, theta, grad, m, v, (long)n, a) != cudaSuccess)
    return POETX_ERR_CUDA;
  return last_launch();
}

poetx_status poetx_adamw_reset(long long n, float* m, float* v, poetx_stream stream) {
  if (n < 0) return POETX_ERR_INVALID_ARG;
  if (n == 0) return POETX_OK;
  POETX_TRY(check_ptrs({m, v}));
  if (cudaMemsetAsync(m, 0, (size_t)n * 4, stream) != cudaSuccess) return POETX_ERR_CUDA;
  return cudaMemsetAsync(v, 0, (size_t)n * 4, stream) == cudaSuccess ? POETX_OK : POETX_ERR_CUDA;
}

poetx_status poetx_check_permutation(const int32_t* perm, int n) {
  if (n < 0 || (n > 0 && perm == nullptr)) return POETX_ERR_INVALID_ARG;
  return is_bijection(perm, n) ? POETX_OK : POETX_ERR_INVALID_ARG;
}

const char* poetx_status_string(poetx_status s) {
  switch (s) {
    case POETX_OK: return "POETX_OK";
    case POETX_ERR_INVALID_ARG: return "POETX_ERR_INVALID_ARG";
    case POETX_ERR_UNSUPPORTED_SHAPE: return "POETX_ERR_UNSUPPORTED_SHAPE";
    case POETX_ERR_ALIGNMENT: return "POETX_ERR_ALIGNMENT";
    case POETX_ERR_WORKSPACE: return "POETX_ERR_WORKSPACE";
    case POETX_ERR_CUDA: return "POETX_ERR_CUDA";
    case POETX_ERR_DEVICE_TIMEOUT: return "POETX_ERR_DEVICE_TIMEOUT";
  }
  return "POETX_ERR_UNKNOWN";
}

size_t poetx_workspace_size(const poetx_desc* desc, int n_tokens) {
  if (check_desc(desc) != POETX_OK || n_tokens < 0) return 0;
  size_t w = cnp_layer_ws(desc);
  w = std::max(w, fwd_plan(desc, n_tokens).total);
  w = std::max(w, bwd_plan(desc, n_tokens).total);
  w = std::max(w, merge_plan(desc).total);
  return w;
}

size_t poetx_cnp_blocks_workspace_size(const poetx_desc* desc, int n_blocks) {
  if (check_desc(desc) != POETX_OK || n_blocks < 0) return 0;
  return cnp_fwd_ws(desc->b, desc->k, desc->dtype, n_blocks);
}

poetx_status poetx_cnp_blocks(const poetx_desc* desc, int n_blocks, const float* theta, void* Q, void* workspace,
                              size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_blocks < 0) return POETX_ERR_INVALID_ARG;
  if (n_blocks == 0) return POETX_OK;
  POETX_TRY(check_ptrs({theta, Q}));
  POETX_TRY(check_ws(workspace, ws_bytes, cnp_fwd_ws(desc->b, desc->k, desc->dtype, n_blocks)));
  return cnp_fwd_run(desc->b, desc->k, desc->dtype, n_blocks, theta, Q, static_cast<char*>(workspace), stream);
}

poetx_status poetx_cnp(const poetx_desc* desc, const float* theta_R, const float* theta_P, void* Q_R, void* Q_P,
                       void* workspace, size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  POETX_TRY(check_ptrs({theta_R, theta_P, Q_R, Q_P}));
  POETX_TRY(check_ws(workspace, ws_bytes, cnp_layer_ws(desc)));
  char* ws = static_cast<char*>(workspace);
  const int b = desc->b;
  const size_t offP = align256(cnp_fwd_ws(b, desc->k, desc->dtype, desc->d_out / b));
  if (cnp_fused_ok(b, desc->dtype)) {
    CnpSide sides[2];
    sides[0].nb = desc->d_out / b; sides[0].theta = theta_R; sides[0].Q = Q_R;
    sides[1].nb = desc->d_in / b; sides[1].theta = theta_P; sides[1].Q = Q_P;
    return cnp_fwd_fused(b, desc->k, sides, 2, stream);
  }
  POETX_TRY(cnp_fwd_generic(b, desc->k, desc->dtype, desc->d_out / b, theta_R, Q_R, ws, stream));
  return cnp_fwd_generic(b, desc->k, desc->dtype, desc->d_in / b, theta_P, Q_P, ws + offP, stream);
}

poetx_status poetx_absorb(const poetx_desc* desc, const void* W0, const int32_t* perm_L, const int32_t* perm_R,
                          void* W0p, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  POETX_TRY(check_ptrs({W0, perm_L, perm_R, W0p}));
  if (W0 == W0p) return POETX_ERR_INVALID_ARG;
  POETX_TRY(debug_check_perms(stream, {{perm_L, desc->d_out}, {perm_R, desc->d_in}}));
  return permute_cols(desc->dtype, W0, desc->d_in, W0p, desc->d_in, desc->d_out, desc->d_in, perm_R, perm_L, false,
                      stream);
}

static poetx_status forward_impl(const poetx_desc* desc, int n_tokens, const void* X, const void* W0p,
                                 const float* W0s, const int32_t* perm_L, const int32_t* perm_R, const void* Q_R,
                                 const void* Q_P, void* Y, void* saved, void* workspace, size_t ws_bytes,
                                 poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_tokens < 0) return POETX_ERR_INVALID_ARG;
  if (n_tokens == 0) return POETX_OK;
  if (desc->mode == POETX_FAST && saved == nullptr) return POETX_ERR_INVALID_ARG;
  if (desc->mode == POETX_MEM && saved != nullptr) return POETX_ERR_INVALID_ARG;
  POETX_TRY(check_ptrs({X, W0p, perm_L, perm_R, Q_R, Q_P, Y}));
  if (saved != nullptr && !aligned16(saved)) return POETX_ERR_ALIGNMENT;
  const FwdPlan f = fwd_plan(desc, n_tokens);
  POETX_TRY(check_ws(workspace, ws_bytes, f.total));
  POETX_TRY(debug_check_perms(stream, {{perm_L, desc->d_out}, {perm_R, desc->d_in}}));
  char* ws = static_cast<char*>(workspace);
  // POET-Xfast keeps Z = V.W0'^T and U = X[:, pi_R] for the backward pass (in `saved`).
  const size_t zbytes = (size_t)n_tokens * desc->d_out * esize(desc->dtype);
  void* Z = desc->mode == POETX_FAST ? saved : ws + f.Z;
  char* U = desc->mode == POETX_FAST ? static_cast<char*>(saved) + zbytes : ws + f.U;
  return forward_chain(desc, n_tokens, X, W0p, W0s, perm_L, perm_R, Q_R, Q_P, Y, Z, U, ws + f.V, ws + f.Yp, stream);
}

poetx_status poetx_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0p,
                           const int32_t* perm_L, const int32_t* perm_R, const void* Q_R, const void* Q_P, void* Y,
                           void* saved, void* workspace, size_t ws_bytes, poetx_stream stream) {
  return forward_impl(desc, n_tokens, X, W0p, nullptr, perm_L, perm_R, Q_R, Q_P, Y, saved, workspace, ws_bytes,
                      stream);
}

// Side stream of the backward pass.  Two chains of the backward are independent: the
// gradient of theta_R's block partials (needs dY' and Z) runs beside dZ -> dV -> dU, and the dX
// scatter (needs dU) runs beside the gradient of theta_P and the CNP adjoint.  They go to a
// per-device non-blocking side stream, ordered with the caller's stream by events only, which
// is also valid under stream capture (the side stream then joins the caller's graph).  A
// per-device mutex keeps concurrent host callers from interleaving the fork and join records.
struct SideStream {
  std::mutex mu;
  cudaStream_t st = nullptr;
  cudaEvent_t ev[4] = {};
  bool ready = false;
};
SideStream g_side[kMaxDevices];

poetx_status side_stream(SideStream** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return POETX_ERR_CUDA;
  SideStream& s = g_side[dev];
  if (!s.ready) {
    if (cudaStreamCreateWithFlags(&s.st, cudaStreamNonBlocking) != cudaSuccess) return POETX_ERR_CUDA;
    for (cudaEvent_t& e : s.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return POETX_ERR_CUDA;
    s.ready = true;
  }
  *out = &s;
  return POETX_OK;
}

// `to` waits for what `from` has enqueued so far.
poetx_status stream_edge(cudaStream_t from, cudaStream_t to, cudaEvent_t e) {
  if (cudaEventRecord(e, from) != cudaSuccess) return POETX_ERR_CUDA;
  return cudaStreamWaitEvent(to, e, 0) == cudaSuccess ? POETX_OK : POETX_ERR_CUDA;
}

// Joins the side stream back into the caller's stream on every exit path once forked.
struct SideJoin {
  cudaStream_t main, side;
  cudaEvent_t e;
  bool armed = false;
  ~SideJoin() {
    if (armed) stream_edge(side, main, e);
  }
};

// CNP and forward pass in one call.  The CNP and the input gather U = X[:, pi_R] are independent
// and neither fills the GPU (the on-chip CNP takes one SM pair per 256-block), so for b = 256
// they run in one launch: the blocks past the CNP pairs gather rows on the remaining SMs.  The
// block-diagonal product, which needs Q_P and U, follows.  Elsewhere the parts run one after
// the other.
poetx_status poetx_cnp_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0p,
                               const int32_t* perm_L, const int32_t* perm_R, const float* theta_R,
                               const float* theta_P, void* Q_R, void* Q_P, void* Y, void* saved, void* workspace,
                               size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  POETX_TRY(check_ptrs({theta_R, theta_P, Q_R, Q_P}));
  const int b = desc->b, dt = desc->dtype;
  if (n_tokens <= 0 || !cnp_fused_ok(b, dt)) {
    if (n_tokens < 0) return POETX_ERR_INVALID_ARG;
    POETX_TRY(poetx_cnp(desc, theta_R, theta_P, Q_R, Q_P, workspace, ws_bytes, stream));
    return forward_impl(desc, n_tokens, X, W0p, nullptr, perm_L, perm_R, Q_R, Q_P, Y, saved, workspace, ws_bytes,
                        stream);
  }
  if (desc->mode == POETX_FAST && saved == nullptr) return POETX_ERR_INVALID_ARG;
  if (desc->mode == POETX_MEM && saved != nullptr) return POETX_ERR_INVALID_ARG;
  POETX_TRY(check_ptrs({X, W0p, perm_L, perm_R, Y}));
  if (saved != nullptr && !aligned16(saved)) return POETX_ERR_ALIGNMENT;
  const FwdPlan f = fwd_plan(desc, n_tokens);
  POETX_TRY(check_ws(workspace, ws_bytes, f.total));
  POETX_TRY(debug_check_perms(stream, {{perm_L, desc->d_out}, {perm_R, desc->d_in}}));
  char* ws = static_cast<char*>(workspace);
  const size_t zbytes = (size_t)n_tokens * desc->d_out * esize(dt);
  void* Z = desc->mode == POETX_FAST ? saved : ws + f.Z;
  char* U = desc->mode == POETX_FAST ? static_cast<char*>(saved) + zbytes : ws + f.U;
  CnpSide sides[2];
  sides[0].nb = desc->d_out / b; sides[0].theta = theta_R; sides[0].Q = Q_R;
  sides[1].nb = desc->d_in / b; sides[1].theta = theta_P; sides[1].Q = Q_P;
  poetx_status st = POETX_OK;
  if (cnp_with_permute<false>(b, desc->k, sides, 2, X, desc->d_in, U, desc->d_in, n_tokens, desc->d_in, perm_R,
                              false, stream, &st)) {
    POETX_TRY(st);
  } else {
    POETX_TRY(cnp_fwd_fused(b, desc->k, sides, 2, stream));
    POETX_TRY(permute_cols(dt, X, desc->d_in, U, desc->d_in, n_tokens, desc->d_in, perm_R, nullptr, false, stream));
  }
  return forward_chain(desc, n_tokens, X, W0p, nullptr, perm_L, perm_R, Q_R, Q_P, Y, Z, U, ws + f.V, ws + f.Yp,
                       stream, true);
}

static poetx_status backward_impl(const poetx_desc* desc, int n_tokens, const void* dY, const void* X,
                                  const void* W0p, const float* W0s, const int32_t* perm_L, const int32_t* perm_R,
                                  const void* Q_R, const void* Q_P, const float* theta_R, const float* theta_P,
                                  const void* saved, void* dX, float* grad_theta_R,
                                  float* grad_theta_P, void* workspace, size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_tokens < 0) return POETX_ERR_INVALID_ARG;
  if (desc->mode == POETX_FAST && saved == nullptr && n_tokens > 0) return POETX_ERR_INVALID_ARG;
  if (desc->mode == POETX_MEM && saved != nullptr) return POETX_ERR_INVALID_ARG;
  POETX_TRY(check_ptrs({theta_R, theta_P, grad_theta_R, grad_theta_P}));
  const int b = desc->b, dt = desc->dtype, nbo = desc->d_out / b, nbi = desc->d_in / b;
  const size_t P = (size_t)b * (b - 1) / 2;
  if (n_tokens == 0) {
    if (cudaMemsetAsync(grad_theta_R, 0, nbo * P * 4, stream) != cudaSuccess) return POETX_ERR_CUDA;
    if (cudaMemsetAsync(grad_theta_P, 0, nbi * P * 4, stream) != cudaSuccess) return POETX_ERR_CUDA;
    return POETX_OK;
  }
  POETX_TRY(check_ptrs({dY, X, W0p, perm_L, perm_R, Q_R, Q_P, dX}));
  if (saved != nullptr && !aligned16(saved)) return POETX_ERR_ALIGNMENT;
  const BwdPlan w = bwd_plan(desc, n_tokens);
  POETX_TRY(check_ws(workspace, ws_bytes, w.total));
  POETX_TRY(debug_check_perms(stream, {{perm_L, desc->d_out}, {perm_R, desc->d_in}}));
  char* ws = static_cast<char*>(workspace);
  const long n = n_tokens;
  const int din = desc->d_in, dout = desc->d_out;

  const void* Z = saved;  // fast mode: Z then U = X[:, pi_R], both kept by the forward pass
  const char* U = desc->mode == POETX_FAST ? static_cast<const char*>(saved) + (size_t)n * dout * esize(dt) : ws + w.U;
  if (desc->mode == POETX_MEM) {
    // POET-Xmem: recompute U = X[:, pi_R], V = BD_P.U and Z = V.W0'^T from X.
    POETX_TRY(forward_chain(desc, n, X, W0p, W0s, perm_L, perm_R, Q_R, Q_P, nullptr, ws + w.Z, ws + w.U, ws + w.V,
                            nullptr, stream));
    Z = ws + w.Z;
  }
  SideStream* ss = nullptr;
  POETX_TRY(side_stream(&ss));
  std::lock_guard<std::mutex> side_lock(ss->mu);
  const cudaStream_t side = ss->st;
  // Output side: dY' = dY[:, pi_L]; then G_R partials on the side stream beside dZ =
  // BD_R^T-adjoint (both read dY', so it is shared through L2), leaving the W0' GEMM below the
  // whole GPU.
  POETX_TRY(permute_cols(dt, dY, dout, ws + w.dYp, dout, n, dout, perm_L, nullptr, false, stream));
  POETX_TRY(bd_backward(dt, n, dout, b, ws + w.dYp, Q_R, ws + w.dZ, stream, true));  // Q_R: from the CNP forward
  POETX_TRY(stream_edge(stream, side, ss->ev[0]));
  SideJoin join{stream, side, ss->ev[3], true};
  // With the on-chip adjoint, G_P's K splits add into one zeroed tile set (the adjoint then reads
  // one partial per block instead of one per split); it is zeroed here, beside the W0' GEMM.
  const bool red_P = cnp_fused_ok(b, dt) && w.sP > 1;
  if (red_P && cudaMemsetAsync(ws + w.GpP, 0, (size_t)nbi * b * b * 4, side) != cudaSuccess) return POETX_ERR_CUDA;
  POETX_TRY(block_grads(dt, n, dout, b, ws + w.dYp, Z, reinterpret_cast<float*>(ws + w.GpR), w.sR, side, w.sR == 1,
                        true));  // Z: saved by the forward or recomputed several launches before
  if (cudaEventRecord(ss->ev[1], side) != cudaSuccess) return POETX_ERR_CUDA;  // G_R partials done
  // dV = dZ . W0' (and, for b = 256, dU_i = dV_i . Q_P,i in the same kernel)
  GemmDesc g;
  g.M = (int)n; g.N = din; g.K = dout;
  g.A = view(ws + w.dZ, n, dout, dout);
  g.B = view(W0p, dout, din, din); g.b_mn = true;
  g.b_scale = W0s;
  g.b_static = true;  // W0' is the caller's, not the output of the launch before (dZ)
  g.epi.d1 = ws + w.dV; g.epi.d1_dtype = dt; g.epi.ld1 = din;
  const bool fused_du = bd_fusable(dt, b, g);
  if (fused_du) POETX_TRY(run_w_gemm(dt, g, Q_P, din, true, ws + w.dU, din, stream, POETX_KC_W_GEMM_ADJ));
  else POETX_TRY(run_w_gemm(dt, g, nullptr, 0, false, nullptr, 0, stream, POETX_KC_W_GEMM_ADJ));
  if (!fused_du) POETX_TRY(bd_backward(dt, n, din, b, ws + w.dV, Q_P, ws + w.dU, stream));
  // Input side: G_P partials (U saved or recomputed), then the CNP adjoint (packed gradients
  // only), which also needs G_R's partials from the side stream.  The scatter dX[:, pi_R] = dU
  // runs in the adjoint's launch on the SMs its pairs leave free (b = 256), else on the side
  // stream from the moment dU exists.
  if (cudaEventRecord(ss->ev[2], stream) != cudaSuccess) return POETX_ERR_CUDA;  // dU done
  if (red_P && cudaStreamWaitEvent(stream, ss->ev[1], 0) != cudaSuccess) return POETX_ERR_CUDA;  // zeroed, G_R done
  POETX_TRY(block_grads(dt, n, din, b, ws + w.dV, U, reinterpret_cast<float*>(ws + w.GpP), w.sP, stream, false,
                        true, red_P));  // U: saved by the forward or recomputed several launches before
  if (!red_P && cudaStreamWaitEvent(stream, ss->ev[1], 0) != cudaSuccess) return POETX_ERR_CUDA;
  CnpSide sides[2];
  sides[0].nb = nbo; sides[0].theta = theta_R; sides[0].part = reinterpret_cast<const float*>(ws + w.GpR);
  sides[0].splits = w.sR; sides[0].grad = grad_theta_R;
  sides[1].nb = nbi; sides[1].theta = theta_P; sides[1].part = reinterpret_cast<const float*>(ws + w.GpP);
  sides[1].splits = red_P ? 1 : w.sP; sides[1].grad = grad_theta_P;
  poetx_status cst = POETX_OK;
  if (cnp_fused_ok(b, dt) &&
      cnp_with_permute<true>(b, desc->k, sides, 2, ws + w.dU, din, dX, din, n, din, perm_R, true, stream, &cst))
    return cst;
  if (cudaStreamWaitEvent(side, ss->ev[2], 0) != cudaSuccess) return POETX_ERR_CUDA;
  POETX_TRY(permute_cols(dt, ws + w.dU, din, dX, din, n, din, perm_R, nullptr, true, side));
  if (cnp_fused_ok(b, dt)) return cnp_bwd_fused(b, desc->k, sides, 2, stream);
  POETX_TRY(cnp_bwd_generic(b, desc->k, dt, nbo, theta_R, reinterpret_cast<const float*>(ws + w.GpR), w.sR,
                            grad_theta_R, ws + w.cnpR, stream));
  return cnp_bwd_generic(b, desc->k, dt, nbi, theta_P, reinterpret_cast<const float*>(ws + w.GpP), w.sP,
                         grad_theta_P, ws + w.cnpP, stream);
}

poetx_status poetx_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* X, const void* W0p,
                            const int32_t* perm_L, const int32_t* perm_R, const void* Q_R, const void* Q_P,
                            const float* theta_R, const float* theta_P, const void* saved,
                            void* dX, float* grad_theta_R, float* grad_theta_P, void* workspace, size_t ws_bytes,
                            poetx_stream stream) {
  return backward_impl(desc, n_tokens, dY, X, W0p, nullptr, perm_L, perm_R, Q_R, Q_P, theta_R, theta_P, saved,
                       dX, grad_theta_R, grad_theta_P, workspace, ws_bytes, stream);
}

size_t poetx_wc_saved_size(const poetx_desc* desc) {
  if (check_desc(desc) != POETX_OK) return 0;
  return 2 * align256((size_t)desc->d_out * desc->d_in * esize(desc->dtype));
}

size_t poetx_wc_workspace_size(const poetx_desc* desc) {
  if (check_desc(desc) != POETX_OK) return 0;
  return std::max(wc_plan(desc).total, cnp_layer_ws(desc));
}

poetx_status poetx_wc_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0p,
                              const int32_t* perm_L, const int32_t* perm_R, const void* Q_R, const void* Q_P, void* Y,
                              void* wc_saved, void* workspace, size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_tokens < 0) return POETX_ERR_INVALID_ARG;
  POETX_TRY(check_ptrs({W0p, perm_L, perm_R, Q_R, Q_P, wc_saved}));
  const WcPlan m = wc_plan(desc);
  POETX_TRY(check_ws(workspace, ws_bytes, m.total));
  char* ws = static_cast<char*>(workspace);
  const int dt = desc->dtype, b = desc->b, din = desc->d_in, dout = desc->d_out;
  char* Wf = static_cast<char*>(wc_saved);
  char* T = Wf + align256((size_t)dout * din * esize(dt));
  {  // T = W0' . BD_P (column blocks)
    GemmDesc g;
    g.M = dout; g.N = b; g.K = b; g.batch = din / b;
    g.A = view(W0p, dout, din, din, 0, b);
    g.B = view(Q_P, din, b, b, b, 0); g.b_mn = true;
    g.epi.d1 = T; g.epi.d1_dtype = dt; g.epi.ld1 = din; g.epi.zcol1 = b;
    POETX_TRY(run_gemm(dt, g, stream, POETX_KC_MERGE_GEMM));
  }
  {  // M = BD_R . T (row blocks)
    GemmDesc g;
    g.M = b; g.N = din; g.K = b; g.batch = dout / b;
    g.A = view(Q_R, dout, b, b, b, 0);
    g.B = view(T, dout, din, din, b, 0); g.b_mn = true;
    g.epi.d1 = ws + m.M2; g.epi.d1_dtype = dt; g.epi.ld1 = din; g.epi.zrow1 = b;
    POETX_TRY(run_gemm(dt, g, stream, POETX_KC_MERGE_GEMM));
  }
  // W[r][c] = M[pi_L^-1(r)][pi_R^-1(c)]
  int32_t* invL = reinterpret_cast<int32_t*>(ws + m.invL);
  int32_t* invR = reinterpret_cast<int32_t*>(ws + m.invR);
  {
    LaunchScope ls(POETX_KC_ELEMENTWISE, stream);
    perm_inverse_kernel<<<ew_grid(dout), 256, 0, stream>>>(perm_L, dout, invL);
  }
  {
    LaunchScope ls(POETX_KC_ELEMENTWISE, stream);
    perm_inverse_kernel<<<ew_grid(din), 256, 0, stream>>>(perm_R, din, invR);
  }
  POETX_TRY(last_launch());
  POETX_TRY(permute_cols(dt, ws + m.M2, din, Wf, din, dout, din, invR, invL, false, stream));
  if (n_tokens == 0) return POETX_OK;
  POETX_TRY(check_ptrs({X, Y}));
  GemmDesc g;  // Y = X . W^T
  g.M = n_tokens; g.N = dout; g.K = din;
  g.A = view(X, n_tokens, din, din);
  g.B = view(Wf, dout, din, din);
  g.epi.d1 = Y; g.epi.d1_dtype = dt; g.epi.ld1 = dout;
  return run_w_gemm(dt, g, nullptr, 0, false, nullptr, 0, stream);
}

poetx_status poetx_wc_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* X, const void* W0p,
                               const int32_t* perm_L, const int32_t* perm_R, const void* Q_R, const float* theta_R,
                               const float* theta_P, const void* wc_saved, void* dX, float* grad_theta_R,
                               float* grad_theta_P, void* workspace, size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_tokens < 1) return POETX_ERR_INVALID_ARG;
  POETX_TRY(check_ptrs({dY, X, W0p, perm_L, perm_R, Q_R, theta_R, theta_P, wc_saved, dX, grad_theta_R, grad_theta_P}));
  const WcPlan m = wc_plan(desc);
  POETX_TRY(check_ws(workspace, ws_bytes, m.total));
  char* ws = static_cast<char*>(workspace);
  const int dt = desc->dtype, b = desc->b, din = desc->d_in, dout = desc->d_out;
  const long n = n_tokens;
  const char* Wf = static_cast<const char*>(wc_saved);
  const char* T = Wf + align256((size_t)dout * din * esize(dt));
  {  // dX = dY . W
    GemmDesc g;
    g.M = (int)n; g.N = din; g.K = dout;
    g.A = view(dY, n, dout, dout);
    g.B = view(Wf, dout, din, din); g.b_mn = true;
    g.epi.d1 = dX; g.epi.d1_dtype = dt; g.epi.ld1 = din;
    POETX_TRY(run_w_gemm(dt, g, nullptr, 0, false, nullptr, 0, stream, POETX_KC_W_GEMM_ADJ));
  }
  {  // dW = dY^T . X  (K = tokens)
    GemmDesc g;
    g.M = dout; g.N = din; g.K = (int)n;
    g.A = view(dY, n, dout, dout); g.a_mn = true;
    g.B = view(X, n, din, din); g.b_mn = true;
    g.epi.d1 = ws + m.dW; g.epi.d1_dtype = dt; g.epi.ld1 = din;
    POETX_TRY(run_gemm(dt, g, stream, POETX_KC_W_GEMM_ADJ));
  }
  // dM[i][j] = dW[pi_L(i)][pi_R(j)]
  POETX_TRY(permute_cols(dt, ws + m.dW, din, ws + m.dM, din, dout, din, perm_R, perm_L, false, stream));
  {  // G_R,i = dM[blk i, :] . T[blk i, :]^T
    GemmDesc g;
    g.M = b; g.N = b; g.K = din; g.batch = dout / b;
    g.A = view(ws + m.dM, dout, din, din, b, 0);
    g.B = view(T, dout, din, din, b, 0);
    g.epi.d1 = ws + m.GpR; g.epi.d1_dtype = F32; g.epi.ld1 = b; g.epi.zrow1 = b;
    POETX_TRY(run_gemm(dt, g, stream, POETX_KC_GRAD_GEMM));
  }
  {  // B1 = BD_R . W0' (row blocks)
    GemmDesc g;
    g.M = b; g.N = din; g.K = b; g.batch = dout / b;
    g.A = view(Q_R, dout, b, b, b, 0);
    g.B = view(W0p, dout, din, din, b, 0); g.b_mn = true;
    g.epi.d1 = ws + m.B1; g.epi.d1_dtype = dt; g.epi.ld1 = din; g.epi.zrow1 = b;
    POETX_TRY(run_gemm(dt, g, stream, POETX_KC_MERGE_GEMM));
  }
  // G_P,j = B1[:, blk j]^T . dM[:, blk j]  (K = d_out rows)
  POETX_TRY(block_grads(dt, dout, din, b, ws + m.B1, ws + m.dM, reinterpret_cast<float*>(ws + m.GpP), 1, stream));
  const int nbo = dout / b, nbi = din / b;
  if (cnp_fused_ok(b, dt)) {
    CnpSide sides[2];
    sides[0].nb = nbo; sides[0].theta = theta_R; sides[0].part = reinterpret_cast<const float*>(ws + m.GpR);
    sides[0].splits = 1; sides[0].grad = grad_theta_R;
    sides[1].nb = nbi; sides[1].theta = theta_P; sides[1].part = reinterpret_cast<const float*>(ws + m.GpP);
    sides[1].splits = 1; sides[1].grad = grad_theta_P;
    return cnp_bwd_fused(b, desc->k, sides, 2, stream);
  }
  POETX_TRY(cnp_bwd_generic(b, desc->k, dt, nbo, theta_R, reinterpret_cast<const float*>(ws + m.GpR), 1, grad_theta_R,
                            ws + m.cnpR, stream));
  return cnp_bwd_generic(b, desc->k, dt, nbi, theta_P, reinterpret_cast<const float*>(ws + m.GpP), 1, grad_theta_P,
                         ws + m.cnpP, stream);
}

// The merge with W0' read from W_in and the new W0' written to W_out (the same array, or for
// POET-XQ the dequantised weight in the M2 region and the result in the T region).
static poetx_status merge_impl(const poetx_desc* desc, const void* W_in, void* W_out, const void* Q_R,
                               const void* Q_P, const int32_t* perm_L_old, const int32_t* perm_R_old,
                               const int32_t* perm_L_new, const int32_t* perm_R_new, float* theta_R, float* theta_P,
                               char* ws, poetx_stream stream) {
  const MergePlan m = merge_plan(desc);
  const int dt = desc->dtype, b = desc->b, din = desc->d_in, dout = desc->d_out;
  // T = W0' . BD_P   (column blocks: T[:, blk z] = W0'[:, blk z] . Q_P,z)
  {
    GemmDesc g;
    g.M = dout; g.N = b; g.K = b; g.batch = din / b;
    g.A = view(W_in, dout, din, din, 0, b);
    g.B = view(Q_P, din, b, b, b, 0); g.b_mn = true;
    g.epi.d1 = ws + m.T; g.epi.d1_dtype = dt; g.epi.ld1 = din; g.epi.zcol1 = b;
    POETX_TRY(run_gemm(dt, g, stream, POETX_KC_MERGE_GEMM));
  }
  // M2 = BD_R . T   (row blocks: M2[blk z, :] = Q_R,z . T[blk z, :])
  {
    GemmDesc g;
    g.M = b; g.N = din; g.K = b; g.batch = dout / b;
    g.A = view(Q_R, dout, b, b, b, 0);
    g.B = view(ws + m.T, dout, din, din, b, 0); g.b_mn = true;
    g.epi.d1 = ws + m.M2; g.epi.d1_dtype = dt; g.epi.ld1 = din; g.epi.zrow1 = b;
    POETX_TRY(run_gemm(dt, g, stream, POETX_KC_MERGE_GEMM));
  }
  // sigma_L = pi_L_old^-1 o pi_L_new, sigma_R likewise; W0'_new[i][j] = M2[sigma_L(i)][sigma_R(j)].
  int32_t* inv = reinterpret_cast<int32_t*>(ws + m.inv);
  int32_t* sL = reinterpret_cast<int32_t*>(ws + m.sigL);
  int32_t* sR = reinterpret_cast<int32_t*>(ws + m.sigR);
  {
    LaunchScope ls(POETX_KC_ELEMENTWISE, stream);
    perm_inverse_kernel<<<ew_grid(dout), 256, 0, stream>>>(perm_L_old, dout, inv);
  }
  {
    LaunchScope ls(POETX_KC_ELEMENTWISE, stream);
    perm_compose_kernel<<<ew_grid(dout), 256, 0, stream>>>(inv, perm_L_new, dout, sL);
  }
  {
    LaunchScope ls(POETX_KC_ELEMENTWISE, stream);
    perm_inverse_kernel<<<ew_grid(din), 256, 0, stream>>>(perm_R_old, din, inv);
  }
  {
    LaunchScope ls(POETX_KC_ELEMENTWISE, stream);
    perm_compose_kernel<<<ew_grid(din), 256, 0, stream>>>(inv, perm_R_new, din, sR);
  }
  POETX_TRY(last_launch());
  POETX_TRY(permute_cols(dt, ws + m.M2, din, W_out, din, dout, din, sR, sL, false, stream));
  const size_t P = (size_t)b * (b - 1) / 2;
  if (cudaMemsetAsync(theta_R, 0, (size_t)(dout / b) * P * 4, stream) != cudaSuccess) return POETX_ERR_CUDA;
  if (cudaMemsetAsync(theta_P, 0, (size_t)(din / b) * P * 4, stream) != cudaSuccess) return POETX_ERR_CUDA;
  return POETX_OK;
}

poetx_status poetx_merge(const poetx_desc* desc, void* W0p, const void* Q_R, const void* Q_P,
                         const int32_t* perm_L_old, const int32_t* perm_R_old, const int32_t* perm_L_new,
                         const int32_t* perm_R_new, float* theta_R, float* theta_P, void* workspace, size_t ws_bytes,
                         poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  POETX_TRY(check_ptrs({W0p, Q_R, Q_P, perm_L_old, perm_R_old, perm_L_new, perm_R_new, theta_R, theta_P}));
  POETX_TRY(check_ws(workspace, ws_bytes, merge_plan(desc).total));
  POETX_TRY(debug_check_perms(stream, {{perm_L_old, desc->d_out}, {perm_R_old, desc->d_in},
                                       {perm_L_new, desc->d_out}, {perm_R_new, desc->d_in}}));
  return merge_impl(desc, W0p, W0p, Q_R, Q_P, perm_L_old, perm_R_old, perm_L_new, perm_R_new, theta_R, theta_P,
                    static_cast<char*>(workspace), stream);
}

// ------------------------------------------------------------------------------- POET-XQ
// POET-XQ holds W0' as int8 codes with one fp32 scale per row and runs POET-Xmem on it: the
// W0' GEMMs dequantise their B tiles in shared memory, nothing keeps a bf16 W0'.
static poetx_status check_xq(const poetx_desc* desc) {
  POETX_TRY(check_desc(desc));
  if (desc->dtype != POETX_BF16 || desc->mode != POETX_MEM) return POETX_ERR_INVALID_ARG;
  if (desc->d_in % 256 || desc->d_out % 256) return POETX_ERR_UNSUPPORTED_SHAPE;
  return POETX_OK;
}

static poetx_status xq_quantize(const poetx_desc* d, const void* W, int8_t* q, float* s, cudaStream_t st) {
  const int grid = (int)std::min<long>((d->d_out + 7) / 8, (long)kNumSms * 8);
  LaunchScope ls(POETX_KC_ELEMENTWISE, st);
  if (launch_pdl(quantize_rows_kernel, dim3(grid), dim3(256), 0, st, static_cast<const uint16_t*>(W), (long)d->d_in,
                 (long)d->d_out, d->d_in, q, (long)d->d_in, s) != cudaSuccess)
    return POETX_ERR_CUDA;
  return last_launch();
}

static poetx_status xq_dequantize(const poetx_desc* d, const int8_t* q, const float* s, void* W, cudaStream_t st) {
  LaunchScope ls(POETX_KC_ELEMENTWISE, st);
  if (launch_pdl(dequantize_rows_kernel, dim3(ew_grid((long)d->d_out * d->d_in / 8)), dim3(256), 0, st, q,
                 (long)d->d_in, s, (long)d->d_out, d->d_in, static_cast<uint16_t*>(W), (long)d->d_in) != cudaSuccess)
    return POETX_ERR_CUDA;
  return last_launch();
}

// --------------------------------------------------------- four-permutation comparator
// The un-absorbed order: R = Pi_L^T BD_R Pi_L and P = Pi_R^T BD_P Pi_R are applied around the
// original W0, so every pass permutes the activations four times (the pages' Table 2 sets this
// against the two-permutation form of poetx_forward / poetx_backward):
//   forward:  U = X[:, pi_R]; V = BD_P.U; Vo[:, pi_R] = V; Z = Vo.W0^T; Z' = Z[:, pi_L];
//             Y' = BD_R.Z'; Y[:, pi_L] = Y'
//   backward: dY' = dY[:, pi_L]; G_R = dY'^T Z'; dZ' = dY'.Q_R; dZ[:, pi_L] = dZ'; dVo = dZ.W0;
//             dV = dVo[:, pi_R]; G_P = dV^T U; dU = dV.Q_P; dX[:, pi_R] = dU; CNP adjoint.
// `saved` keeps Z' then U (as POET-Xfast's `saved`) from the forward for the backward.
struct FpPlan {
  size_t V, Vo, Z, Yp, dYp, dZp, dZ, dVo, dV, dU, GpR, GpP, cnpR, cnpP, total;
  int sR, sP;
};
FpPlan fp_plan(const poetx_desc* d, long n) {
  const size_t e = esize(d->dtype);
  const int b = d->b, nbo = d->d_out / b, nbi = d->d_in / b;
  FpPlan f;
  Plan p;
  f.V = p.take(n * d->d_in * e);
  f.Vo = p.take(n * d->d_in * e);
  f.Z = p.take(n * d->d_out * e);
  f.Yp = p.take(n * d->d_out * e);
  f.dYp = p.take(n * d->d_out * e);
  f.dZp = p.take(n * d->d_out * e);
  f.dZ = p.take(n * d->d_out * e);
  f.dVo = p.take(n * d->d_in * e);
  f.dV = p.take(n * d->d_in * e);
  f.dU = p.take(n * d->d_in * e);
  f.sR = grad_splits(d->dtype, n, nbo, b);
  f.sP = grad_splits(d->dtype, n, nbi, b);
  f.GpR = p.take((size_t)f.sR * nbo * b * b * 4);
  f.GpP = p.take((size_t)f.sP * nbi * b * b * 4);
  f.cnpR = p.take(cnp_bwd_ws(b, d->k, d->dtype, nbo));
  f.cnpP = p.take(cnp_bwd_ws(b, d->k, d->dtype, nbi));
  f.total = p.total;
  return f;
}

size_t poetx_fourperm_workspace_size(const poetx_desc* desc, int n_tokens) {
  if (check_desc(desc) != POETX_OK || n_tokens < 0) return 0;
  return std::max(fp_plan(desc, n_tokens).total, cnp_layer_ws(desc));
}

poetx_status poetx_fourperm_forward(const poetx_desc* desc, int n_tokens, const void* X, const void* W0,
                                    const int32_t* perm_L, const int32_t* perm_R, const void* Q_R, const void* Q_P,
                                    void* Y, void* saved, void* workspace, size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_tokens < 0) return POETX_ERR_INVALID_ARG;
  if (n_tokens == 0) return POETX_OK;
  POETX_TRY(check_ptrs({X, W0, perm_L, perm_R, Q_R, Q_P, Y, saved}));
  const FpPlan f = fp_plan(desc, n_tokens);
  POETX_TRY(check_ws(workspace, ws_bytes, f.total));
  char* ws = static_cast<char*>(workspace);
  const int dt = desc->dtype, b = desc->b, din = desc->d_in, dout = desc->d_out;
  const long n = n_tokens;
  char* Zp = static_cast<char*>(saved);
  char* U = Zp + (size_t)n * dout * esize(dt);
  POETX_TRY(permute_cols(dt, X, din, U, din, n, din, perm_R, nullptr, false, stream));
  POETX_TRY(bd_forward(dt, n, din, b, U, Q_P, ws + f.V, stream));
  POETX_TRY(permute_cols(dt, ws + f.V, din, ws + f.Vo, din, n, din, perm_R, nullptr, true, stream));
  GemmDesc g;
  g.M = (int)n; g.N = dout; g.K = din;
  g.A = view(ws + f.Vo, n, din, din);
  g.B = view(W0, dout, din, din);
  g.epi.d1 = ws + f.Z; g.epi.d1_dtype = dt; g.epi.ld1 = dout;
  POETX_TRY(run_w_gemm(dt, g, nullptr, 0, false, nullptr, 0, stream));
  POETX_TRY(permute_cols(dt, ws + f.Z, dout, Zp, dout, n, dout, perm_L, nullptr, false, stream));
  POETX_TRY(bd_forward(dt, n, dout, b, Zp, Q_R, ws + f.Yp, stream));
  return permute_cols(dt, ws + f.Yp, dout, Y, dout, n, dout, perm_L, nullptr, true, stream);
}

poetx_status poetx_fourperm_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* W0,
                                     const int32_t* perm_L, const int32_t* perm_R, const void* Q_R, const void* Q_P,
                                     const float* theta_R, const float* theta_P, const void* saved, void* dX,
                                     float* grad_theta_R, float* grad_theta_P, void* workspace, size_t ws_bytes,
                                     poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_tokens < 0) return POETX_ERR_INVALID_ARG;
  POETX_TRY(check_ptrs({theta_R, theta_P, grad_theta_R, grad_theta_P}));
  const int b = desc->b, dt = desc->dtype, din = desc->d_in, dout = desc->d_out, nbo = dout / b, nbi = din / b;
  if (n_tokens == 0) {
    const size_t P = (size_t)b * (b - 1) / 2;
    if (cudaMemsetAsync(grad_theta_R, 0, nbo * P * 4, stream) != cudaSuccess) return POETX_ERR_CUDA;
    return cudaMemsetAsync(grad_theta_P, 0, nbi * P * 4, stream) == cudaSuccess ? POETX_OK : POETX_ERR_CUDA;
  }
  POETX_TRY(check_ptrs({dY, W0, perm_L, perm_R, Q_R, Q_P, saved, dX}));
  const FpPlan f = fp_plan(desc, n_tokens);
  POETX_TRY(check_ws(workspace, ws_bytes, f.total));
  char* ws = static_cast<char*>(workspace);
  const long n = n_tokens;
  const char* Zp = static_cast<const char*>(saved);
  const char* U = Zp + (size_t)n * dout * esize(dt);
  POETX_TRY(permute_cols(dt, dY, dout, ws + f.dYp, dout, n, dout, perm_L, nullptr, false, stream));
  POETX_TRY(block_grads(dt, n, dout, b, ws + f.dYp, Zp, reinterpret_cast<float*>(ws + f.GpR), f.sR, stream));
  POETX_TRY(bd_backward(dt, n, dout, b, ws + f.dYp, Q_R, ws + f.dZp, stream));
  POETX_TRY(permute_cols(dt, ws + f.dZp, dout, ws + f.dZ, dout, n, dout, perm_L, nullptr, true, stream));
  GemmDesc g;
  g.M = (int)n; g.N = din; g.K = dout;
  g.A = view(ws + f.dZ, n, dout, dout);
  g.B = view(W0, dout, din, din); g.b_mn = true;
  g.epi.d1 = ws + f.dVo; g.epi.d1_dtype = dt; g.epi.ld1 = din;
  POETX_TRY(run_w_gemm(dt, g, nullptr, 0, false, nullptr, 0, stream, POETX_KC_W_GEMM_ADJ));
  POETX_TRY(permute_cols(dt, ws + f.dVo, din, ws + f.dV, din, n, din, perm_R, nullptr, false, stream));
  POETX_TRY(block_grads(dt, n, din, b, ws + f.dV, U, reinterpret_cast<float*>(ws + f.GpP), f.sP, stream));
  POETX_TRY(bd_backward(dt, n, din, b, ws + f.dV, Q_P, ws + f.dU, stream));
  POETX_TRY(permute_cols(dt, ws + f.dU, din, dX, din, n, din, perm_R, nullptr, true, stream));
  if (cnp_fused_ok(b, dt)) {
    CnpSide sides[2];
    sides[0].nb = nbo; sides[0].theta = theta_R; sides[0].part = reinterpret_cast<const float*>(ws + f.GpR);
    sides[0].splits = f.sR; sides[0].grad = grad_theta_R;
    sides[1].nb = nbi; sides[1].theta = theta_P; sides[1].part = reinterpret_cast<const float*>(ws + f.GpP);
    sides[1].splits = f.sP; sides[1].grad = grad_theta_P;
    return cnp_bwd_fused(b, desc->k, sides, 2, stream);
  }
  POETX_TRY(cnp_bwd_generic(b, desc->k, dt, nbo, theta_R, reinterpret_cast<const float*>(ws + f.GpR), f.sR,
                            grad_theta_R, ws + f.cnpR, stream));
  return cnp_bwd_generic(b, desc->k, dt, nbi, theta_P, reinterpret_cast<const float*>(ws + f.GpP), f.sP,
                         grad_theta_P, ws + f.cnpP, stream);
}

poetx_status poetx_xq_quantize(const poetx_desc* desc, const void* W0p, int8_t* W0q, float* W0s,
                               poetx_stream stream) {
  POETX_TRY(check_xq(desc));
  POETX_TRY(check_ptrs({W0p, W0q, W0s}));
  return xq_quantize(desc, W0p, W0q, W0s, stream);
}

poetx_status poetx_xq_dequantize(const poetx_desc* desc, const int8_t* W0q, const float* W0s, void* W0p,
                                 poetx_stream stream) {
  POETX_TRY(check_xq(desc));
  POETX_TRY(check_ptrs({W0p, W0q, W0s}));
  return xq_dequantize(desc, W0q, W0s, W0p, stream);
}

poetx_status poetx_xq_forward(const poetx_desc* desc, int n_tokens, const void* X, const int8_t* W0q,
                              const float* W0s, const int32_t* perm_L, const int32_t* perm_R, const void* Q_R,
                              const void* Q_P, void* Y, void* workspace, size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_xq(desc));
  POETX_TRY(check_ptrs({W0q, W0s}));
  return forward_impl(desc, n_tokens, X, W0q, W0s, perm_L, perm_R, Q_R, Q_P, Y, nullptr, workspace, ws_bytes,
                      stream);
}

poetx_status poetx_xq_backward(const poetx_desc* desc, int n_tokens, const void* dY, const void* X,
                               const int8_t* W0q, const float* W0s, const int32_t* perm_L, const int32_t* perm_R,
                               const void* Q_R, const void* Q_P, const float* theta_R, const float* theta_P,
                               void* dX, float* grad_theta_R, float* grad_theta_P, void* workspace, size_t ws_bytes,
                               poetx_stream stream) {
  POETX_TRY(check_xq(desc));
  POETX_TRY(check_ptrs({W0q, W0s}));
  return backward_impl(desc, n_tokens, dY, X, W0q, W0s, perm_L, perm_R, Q_R, Q_P, theta_R, theta_P, nullptr,
                       dX, grad_theta_R, grad_theta_P, workspace, ws_bytes, stream);
}

poetx_status poetx_xq_merge(const poetx_desc* desc, int8_t* W0q, float* W0s, const void* Q_R, const void* Q_P,
                            const int32_t* perm_L_old, const int32_t* perm_R_old, const int32_t* perm_L_new,
                            const int32_t* perm_R_new, float* theta_R, float* theta_P, void* workspace,
                            size_t ws_bytes, poetx_stream stream) {
  POETX_TRY(check_xq(desc));
  POETX_TRY(check_ptrs({W0q, W0s, Q_R, Q_P, perm_L_old, perm_R_old, perm_L_new, perm_R_new, theta_R, theta_P}));
  const MergePlan m = merge_plan(desc);
  POETX_TRY(check_ws(workspace, ws_bytes, m.total));
  char* ws = static_cast<char*>(workspace);
  // Dequantise into the M2 region (read only by the first merge product), merge into the T
  // region, quantise back.  The bf16 weight lives only in the workspace for the call.
  POETX_TRY(xq_dequantize(desc, W0q, W0s, ws + m.M2, stream));
  POETX_TRY(merge_impl(desc, ws + m.M2, ws + m.T, Q_R, Q_P, perm_L_old, perm_R_old, perm_L_new, perm_R_new, theta_R,
                       theta_P, ws, stream));
  return xq_quantize(desc, ws + m.T, W0q, W0s, stream);
}

poetx_status poetx_device_status(int* detail) {
  if (cudaDeviceSynchronize() != cudaSuccess) return POETX_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return POETX_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return POETX_ERR_CUDA;
  if (detail) *detail = v;
  return v ? POETX_ERR_DEVICE_TIMEOUT : POETX_OK;
}

// Failure-detection probe: one CTA waits on a shared-memory mbarrier that nothing ever arrives
// on, bounded by limit_ns.  The bounded wait gives up, records (KID_WAIT_PROBE, 1) in the device
// error word and returns; the kernel then writes 2 to *returned (1 would mean the wait completed).
enum : int { KID_WAIT_PROBE = 7 };
__global__ void wait_probe_kernel(unsigned long long limit_ns, int* returned) {
  using namespace sm100;
  __shared__ uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool done = mbar_wait_limit(b, 0, limit_ns, KID_WAIT_PROBE, 1);
  __syncthreads();
  if (threadIdx.x == 0) *returned = done ? 1 : 2;
}

poetx_status poetx_test_wait_timeout(long long limit_ns, int* returned, poetx_stream stream) {
  if (returned == nullptr || limit_ns < 1000 || limit_ns > 100000000LL) return POETX_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(returned) & 3u) != 0) return POETX_ERR_ALIGNMENT;
  LaunchScope ls(POETX_KC_ELEMENTWISE, stream);
  wait_probe_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_ns, returned);
  return last_launch();
}

poetx_status poetx_test_gemm(int dtype, int M, int N, int K, int batch, int splits, const void* a, long long a_rows,
                             long long a_cols, long long a_ld, long long a_zrow, long long a_zcol, int a_mn,
                             const void* b, long long b_rows, long long b_cols, long long b_ld, long long b_zrow,
                             long long b_zcol, int b_mn, void* d, int d_dtype, long long d_ld, long long d_zrow,
                             long long d_zcol, long long d_split_stride, float alpha, float beta, const float* c,
                             long long c_ld, long long c_zrow, long long c_zcol, int diag, poetx_stream stream) {
  if (dtype != F32 && dtype != BF16) return POETX_ERR_INVALID_ARG;
  if (d_dtype != F32 && d_dtype != BF16) return POETX_ERR_INVALID_ARG;
  if (d == nullptr) return POETX_ERR_INVALID_ARG;
  GemmDesc g;
  g.M = M; g.N = N; g.K = K; g.batch = batch; g.splits = splits;
  g.A = view(a, a_rows, a_cols, a_ld, a_zrow, a_zcol); g.a_mn = a_mn != 0;
  g.B = view(b, b_rows, b_cols, b_ld, b_zrow, b_zcol); g.b_mn = b_mn != 0;
  g.epi.d1 = d; g.epi.d1_dtype = d_dtype; g.epi.ld1 = d_ld; g.epi.zrow1 = d_zrow; g.epi.zcol1 = d_zcol;
  g.epi.split_stride1 = d_split_stride; g.epi.alpha1 = alpha; g.epi.beta1 = beta; g.epi.diag1 = diag;
  g.epi.c = c; g.epi.c_dtype = F32; g.epi.ldc = c_ld; g.epi.zrowc = c_zrow; g.epi.zcolc = c_zcol;
  return run_gemm(dtype, g, stream, POETX_KC_TEST_GEMM);
}

unsigned long long poetx_launch_count(void) { return prof().launches.load(); }

poetx_status poetx_profile_enable(int on) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (on) {
    p.recs.clear();
    p.used = 0;
  }
  p.on = on != 0;
  return POETX_OK;
}

poetx_status poetx_profile_summary(int* counts, float* total_ms) {
  if (counts == nullptr || total_ms == nullptr) return POETX_ERR_INVALID_ARG;
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (int c = 0; c < POETX_KC_COUNT; ++c) { counts[c] = 0; total_ms[c] = 0.f; }
  for (auto& r : p.recs) {
    if (cudaEventSynchronize(r.second.second) != cudaSuccess) return POETX_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.second.first, r.second.second) != cudaSuccess) return POETX_ERR_CUDA;
    if (r.first >= 0 && r.first < POETX_KC_COUNT) { counts[r.first] += 1; total_ms[r.first] += ms; }
  }
  return POETX_OK;
}

poetx_status poetx_cnp_blocks_noalloc(const poetx_desc* desc, int n_blocks, const float* theta, void* Q,
                                      poetx_stream stream) {
  POETX_TRY(check_desc(desc));
  if (n_blocks < 0) return POETX_ERR_INVALID_ARG;
  if (n_blocks == 0) return POETX_OK;
  POETX_TRY(check_ptrs({theta, Q}));
  if (cnp_fwd_ws(desc->b, desc->k, desc->dtype, n_blocks) > kNoAllocScratchBytes) return POETX_ERR_WORKSPACE;
  char* ws = nullptr;
  POETX_TRY(noalloc_scratch(&ws));
  return cnp_fwd_run(desc->b, desc->k, desc->dtype, n_blocks, theta, Q, ws, stream);
}

}  // extern "C"
