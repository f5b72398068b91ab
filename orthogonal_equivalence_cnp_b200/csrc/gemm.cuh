// Batched GEMM core of the POET-X layer.
//
// Every contraction of the layer — the block-diagonal products BD_P·x and BD_R·z (replication
// review of POET-X, "Summary": batch-parallel block-diagonal matmul that never builds the
// sparse matrix), the W0' products, the per-block gradient products, the Cayley–Neumann
// power products and the merge — is one call of
//
//     D[z][m][n] = sum_k A[z][m][k] * B[z][n][k]          z < batch, m < M, n < N
//
// where A and B are views of row-major 2-D arrays.  A view is (base, rows, cols, ld) plus a
// per-batch coordinate offset (zrow, zcol); "K-major" means A[z][m][k] = mem[z*zrow+m][z*zcol+k]
// and "MN-major" means A[z][m][k] = mem[z*zrow+k][z*zcol+m] (likewise for B with n).  Split-K
// writes one partial result per split.  The epilogue is
//
//     D1 = alpha1*acc + beta1*C (+ I if diag1)          (bf16 or f32, partial `split` offset)
//     D2 = alpha2*acc + beta2*C (+ D2 if accum2)        (f32)
//
// with an optional addend C.  The bf16 path runs on tcgen05 tensor cores (fp32 accumulation in
// TMEM, operands staged by TMA into 128-byte-swizzled shared memory); the f32 path runs on the
// CUDA cores in plain fp32 FMA (no tf32), for the fp32 workloads.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace poetx {

struct Operand {
  const void* base = nullptr;
  long rows = 0, cols = 0, ld = 0;  // extent and row stride of the whole 2-D array (elements)
  long zrow = 0, zcol = 0;          // coordinate offset per batch index
};

struct Epilogue {
  void* d1 = nullptr;
  long ld1 = 0, zrow1 = 0, zcol1 = 0, split_stride1 = 0;
  int d1_dtype = F32;
  float alpha1 = 1.f, beta1 = 0.f;
  int diag1 = 0;
  int red1 = 0;  // f32 d1 only: added into d1 (red.global.add) instead of stored; every split adds into the same tile
  float* d2 = nullptr;
  long ld2 = 0, zrow2 = 0, zcol2 = 0;
  float alpha2 = 1.f, beta2 = 0.f;
  int accum2 = 0;
  const void* c = nullptr;
  long ldc = 0, zrowc = 0, zcolc = 0;
  int c_dtype = F32;
};

struct GemmDesc {
  int M = 0, N = 0, K = 0, batch = 1, splits = 1;
  Operand A, B;
  bool a_mn = false, b_mn = false;
  Epilogue epi;
  const float* b_scale = nullptr;  // set: B is int8 codes, B row r scaled by b_scale[r] (W0' GEMM only)
  // B was not written by the kernel launched just before this one (W0' GEMM only): its first
  // stages may be requested before the wait for that kernel.
  bool b_static = false;
};

// Kernel ids recorded in the device error word.
enum KernelId : int { KID_GEMM_TC = 1 };

// ------------------------------------------------------------------------------- epilogue
__device__ __forceinline__ void load32(const void* base, long off, int dt, float (&v)[32]) {
  if (dt == BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + off);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = p[q];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        v[q * 8 + 2 * t] = __uint_as_float(w[t] << 16);
        v[q * 8 + 2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 f = p[q];
      v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void store32(void* base, long off, int dt, const float (&v)[32]) {
  if (dt == BF16) {
    uint4* p = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + off);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      p[q] = make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]), pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                        pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]), pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]));
  } else {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + off);
#pragma unroll
    for (int q = 0; q < 8; ++q) p[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  }
}

// Loads the 32 addend values of row m, columns n..n+31 (batch z).
__device__ __forceinline__ void epilogue_load_c(const Epilogue& e, int z, int m, int n, float (&cv)[32]) {
  if (e.c != nullptr) load32(e.c, ((long)z * e.zrowc + m) * e.ldc + (long)z * e.zcolc + n, e.c_dtype, cv);
}

// Applies the epilogue to 32 consecutive columns n..n+31 of row m (batch z, split `split`),
// with the addend values already in cv.
__device__ __forceinline__ void epilogue32c(const Epilogue& e, int z, int split, int m, int n,
                                            const float (&acc)[32], const float (&cv)[32]) {
  const bool has_c = e.c != nullptr;
  if (e.d1 != nullptr) {
    float o[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float v = e.alpha1 * acc[j];
      if (has_c) v += e.beta1 * cv[j];
      if (e.diag1 && m == n + j) v += 1.f;
      o[j] = v;
    }
    const long off = ((long)z * e.zrow1 + m) * e.ld1 + (long)z * e.zcol1 + n + (long)split * e.split_stride1;
    if (e.red1) {
      float* p = reinterpret_cast<float*>(e.d1) + off;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p + 4 * q), "f"(o[4 * q]), "f"(o[4 * q + 1]),
                     "f"(o[4 * q + 2]), "f"(o[4 * q + 3])
                     : "memory");
    } else {
      store32(e.d1, off, e.d1_dtype, o);
    }
  }
  if (e.d2 != nullptr) {
    const long off = ((long)z * e.zrow2 + m) * e.ld2 + (long)z * e.zcol2 + n;
    float o[32];
    if (e.accum2) load32(e.d2, off, F32, o);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float v = e.alpha2 * acc[j];
      if (has_c) v += e.beta2 * cv[j];
      o[j] = e.accum2 ? o[j] + v : v;
    }
    store32(e.d2, off, F32, o);
  }
}

__device__ __forceinline__ void epilogue32(const Epilogue& e, int z, int split, int m, int n,
                                           const float (&acc)[32]) {
  float cv[32];
  epilogue_load_c(e, z, m, n, cv);
  epilogue32c(e, z, split, m, n, acc, cv);
}

// Drains a BN-column TMEM accumulator (this thread's lane = tile row m) through the epilogue,
// loading the addend of the next 32-column chunk before storing the current one.
template <int BN>
__device__ __forceinline__ void drain_tile(uint32_t taddr, const Epilogue& e, int z, int split, int m, bool row_ok,
                                           int n0, bool zero_acc) {
  float cv[32], cn[32];
  if (row_ok) epilogue_load_c(e, z, m, n0, cv);
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    uint32_t r[32];
    sm100::tmem_ld_32x32b_x32(taddr + (uint32_t)c, r);
    sm100::tmem_wait_ld();
    if (row_ok && c + 32 < BN) epilogue_load_c(e, z, m, n0 + c + 32, cn);
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = zero_acc ? 0.f : __uint_as_float(r[j]);
    if (row_ok) epilogue32c(e, z, split, m, n0 + c, acc, cv);
#pragma unroll
    for (int j = 0; j < 32; ++j) cv[j] = cn[j];
  }
}

__device__ __forceinline__ void epilogue1(const Epilogue& e, int z, int split, int m, int n, float acc) {
  float c = 0.f;
  if (e.c != nullptr) c = load_elem(e.c, ((long)z * e.zrowc + m) * e.ldc + (long)z * e.zcolc + n, e.c_dtype);
  if (e.d1 != nullptr) {
    float v = e.alpha1 * acc + e.beta1 * c + ((e.diag1 && m == n) ? 1.f : 0.f);
    const long off = ((long)z * e.zrow1 + m) * e.ld1 + (long)z * e.zcol1 + n + (long)split * e.split_stride1;
    if (e.red1) atomicAdd(reinterpret_cast<float*>(e.d1) + off, v);
    else store_elem(e.d1, off, e.d1_dtype, v);
  }
  if (e.d2 != nullptr) {
    const long off = ((long)z * e.zrow2 + m) * e.ld2 + (long)z * e.zcol2 + n;
    float v = e.alpha2 * acc + e.beta2 * c;
    e.d2[off] = e.accum2 ? e.d2[off] + v : v;
  }
}

// ------------------------------------------------------------------------ tcgen05 kernel
struct TcArgs {
  int M, N, K, splits;
  int a_zrow, a_zcol, b_zrow, b_zcol;
  int tma_store;  // plain bf16 d1 (no addend/alpha/diag/d2/splits, zrow1 = 0): TMA-store epilogue
  int b_early;    // B is not the previous launch's output: its first stages are requested before the wait
  Epilogue epi;
};

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;  // 64 bf16 = 128 B = one swizzle span

template <int BN, int STAGES>
__host__ __device__ constexpr size_t tc_smem_bytes() {
  return (size_t)STAGES * (TC_BM * TC_BK * 2 + BN * TC_BK * 2) + 1024 /*align*/ + 256 /*barriers*/;
}

// One CTA computes one BM x BN output tile of one (batch, split).  Warp 0 lane 0 streams A/B
// k-tiles with TMA into a STAGES-deep ring; warp 1 lane 0 issues tcgen05.mma (M=128, N=BN,
// K=16) into a TMEM accumulator of BN fp32 columns and frees ring slots with tcgen05.commit;
// then all four warps drain TMEM (warp w owns TMEM lanes 32w..32w+31 = tile rows) through the
// epilogue.  Every wait is bounded (kWaitLimitNs); on a timeout the CTA records the error,
// skips the rest of its work and still releases its TMEM.
template <int BN, int STAGES, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(128)
    gemm_bf16_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmD, const TcArgs args) {
  constexpr uint32_t A_BYTES = TC_BM * TC_BK * 2;
  constexpr uint32_t B_BYTES = BN * TC_BK * 2;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t IDESC = sm100::idesc_bf16_f32(TC_BM, BN, A_MN, B_MN);
  using namespace sm100;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  const uint32_t smem0 = smem_u32(smem);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  const uint32_t accum_bar = smem_u32(bars + 2 * STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int z = blockIdx.z / args.splits, split = blockIdx.z % args.splits;
  const int m0 = blockIdx.y * TC_BM, n0 = blockIdx.x * BN;
  const int KT = (args.K + TC_BK - 1) / TC_BK;
  const int kt0 = (int)((long)KT * split / args.splits);
  const int kt1 = (int)((long)KT * (split + 1) / args.splits);
  const int nkt = kt1 - kt0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accum_bar, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_holder;
  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    auto load_b = [&](int i, int s) {
      const int k0 = (kt0 + i) * TC_BK;
      const uint32_t sb = smem0 + s * STAGE_BYTES + A_BYTES;
      if (!B_MN) {
        tma_load_2d(sb, &tmB, full_bar(s), z * args.b_zcol + k0, z * args.b_zrow + n0);
      } else {
#pragma unroll
        for (int h = 0; h < BN / 64; ++h)
          tma_load_2d(sb + h * 8192, &tmB, full_bar(s), z * args.b_zcol + n0 + 64 * h, z * args.b_zrow + k0);
      }
    };
    // B of the first stages while the previous kernel (which wrote A) finishes.
    const int early = args.b_early ? min(nkt, STAGES) : 0;
    for (int i = 0; i < early; ++i) {
      mbar_arrive_expect_tx(full_bar(i), STAGE_BYTES);
      load_b(i, i);
    }
    griddep_wait();  // A and the epilogue's addends may come from the previous kernel
    for (int i = 0; i < nkt; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      if (i >= early) {
        if (!mbar_wait(empty_bar(s), ph ^ 1u, KID_GEMM_TC, 1)) break;
        mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES);
        load_b(i, s);
      }
      const int k0 = (kt0 + i) * TC_BK;
      const uint32_t sa = smem0 + s * STAGE_BYTES;
      if (!A_MN) {
        tma_load_2d(sa, &tmA, full_bar(s), z * args.a_zcol + k0, z * args.a_zrow + m0);
      } else {
#pragma unroll
        for (int h = 0; h < TC_BM / 64; ++h)
          tma_load_2d(sa + h * 8192, &tmA, full_bar(s), z * args.a_zcol + m0 + 64 * h, z * args.a_zrow + k0);
      }
    }
  } else {
    griddep_wait();  // operands and epilogue addends may come from the previous kernel
  }
  if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    for (int i = 0; i < nkt; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      if (!mbar_wait(full_bar(s), ph, KID_GEMM_TC, 2)) break;
      tc_fence_after();
      const uint32_t sa = smem0 + s * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk) {
        const uint64_t ad = A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024) : smem_desc_sw128(sa + kk * 32, 16, 1024);
        const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
        mma_bf16(tmem_d, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(empty_bar(s));
    }
    mma_commit(accum_bar);
  }
  __syncwarp();

  // ---------------- epilogue: TMEM -> registers -> global
  bool ok = mbar_wait(accum_bar, 0, KID_GEMM_TC, 3);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  griddep_launch();
  if (ok && args.tma_store) {
    // Each warp stages its 32 rows x 64 columns as a 128-byte-swizzled box (two 4 KiB buffers
    // per warp in the idle ring) and lane 0 stores it with TMA: whole lines instead of one
    // 16-byte piece per row, and rows past M are clipped by the map.
    const uint32_t taddr = tmem_d + ((uint32_t)(warp * 32) << 16);
    const Epilogue& e = args.epi;
#pragma unroll 1
    for (int c64 = 0; c64 < BN / 64; ++c64) {
      uint8_t* buf = smem + warp * 8192 + (c64 & 1) * 4096;
      if (c64 >= 2) {
        if (lane == 0) bulk_wait_read<1>();  // the store two boxes back has read this buffer
        __syncwarp();
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + (uint32_t)(c64 * 64 + hh * 32), v);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = 8 * u;
          const float f0 = nkt == 0 ? 0.f : __uint_as_float(v[j]), f1 = nkt == 0 ? 0.f : __uint_as_float(v[j + 1]);
          const float f2 = nkt == 0 ? 0.f : __uint_as_float(v[j + 2]), f3 = nkt == 0 ? 0.f : __uint_as_float(v[j + 3]);
          const float f4 = nkt == 0 ? 0.f : __uint_as_float(v[j + 4]), f5 = nkt == 0 ? 0.f : __uint_as_float(v[j + 5]);
          const float f6 = nkt == 0 ? 0.f : __uint_as_float(v[j + 6]), f7 = nkt == 0 ? 0.f : __uint_as_float(v[j + 7]);
          const uint4 q = make_uint4(pack_bf16x2(f0, f1), pack_bf16x2(f2, f3), pack_bf16x2(f4, f5), pack_bf16x2(f6, f7));
          const int ch = hh * 4 + u;
          *reinterpret_cast<uint4*>(buf + lane * 128 + ((ch ^ (lane & 7)) * 16)) = q;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tmD, smem_u32(buf), (int)(z * e.zcol1) + n0 + c64 * 64, m0 + warp * 32);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_read<0>();
  } else if (ok) {
    const int m = m0 + warp * 32 + lane;
    drain_tile<BN>(tmem_d + ((uint32_t)(warp * 32) << 16), args.epi, z, split, m, m < args.M, n0, nkt == 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_d, BN);
}

// ------------------------------------------------- W0' GEMM fused with a block-diagonal factor
// One 128 x 256 output tile of D = A . B^T (A K-major, B K- or MN-major) where the 256 columns
// are exactly one b = 256 block; after the K loop the tile is (a) stored (bf16, optional) and
// (b) written as bf16 into the idle TMA ring in the 128-byte-swizzled K-major layout, where it
// is the A operand of a second tcgen05 product with that block's Q (K-major: out2 = D . Q^T,
// forward BD_R; MN-major: out2 = D . Q, adjoint of BD_P).  Two accumulators share TMEM
// (columns 0..255 and 256..511).  This removes a separate block-diagonal launch and its read
// of D.  All waits bounded; every thread reaches every barrier.
struct FuseArgs {
  int M, N, K;
  void* d1;       // bf16 [M, N] store of D (may be null)
  long ld1;
  void* out2;     // bf16 [M, N] result of the block-diagonal factor
  long ld2;
};

template <bool B_MN, bool Q_MN>
__global__ void __launch_bounds__(128, 1)
    gemm_bd_fused_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmQ, const FuseArgs args) {
  constexpr int BN = 256, STAGES = 4;
  constexpr uint32_t A_BYTES = TC_BM * TC_BK * 2;
  constexpr uint32_t B_BYTES = BN * TC_BK * 2;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t IDESC = sm100::idesc_bf16_f32(TC_BM, BN, false, B_MN);
  constexpr uint32_t IDESC2 = sm100::idesc_bf16_f32(TC_BM, BN, false, Q_MN);
  using namespace sm100;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 3);
  const uint32_t smem0 = smem_u32(smem);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  const uint32_t accum_bar = smem_u32(bars + 2 * STAGES);
  const uint32_t q_full = smem_u32(bars + 2 * STAGES + 1);
  const uint32_t acc2_bar = smem_u32(bars + 2 * STAGES + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * TC_BM, n0 = blockIdx.x * BN;
  const int zq = blockIdx.x;  // the b = 256 block this tile's columns form
  const int nkt = (args.K + TC_BK - 1) / TC_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accum_bar, 1);
    mbar_init(q_full, 1);
    mbar_init(acc2_bar, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmQ);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_holder;
  griddep_wait();

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer: the K loop, then this block's Q into the ring's B halves.
    bool ok = true;
    for (int i = 0; i < nkt; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      if (!mbar_wait(empty_bar(s), ph ^ 1u, KID_GEMM_TC, 5)) { ok = false; break; }
      mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES);
      const int k0 = i * TC_BK;
      const uint32_t sa = smem0 + s * STAGE_BYTES, sb = sa + A_BYTES;
      tma_load_2d(sa, &tmA, full_bar(s), k0, m0);
      if (!B_MN) {
        tma_load_2d(sb, &tmB, full_bar(s), k0, n0);
      } else {
#pragma unroll
        for (int h = 0; h < BN / 64; ++h) tma_load_2d(sb + h * 8192, &tmB, full_bar(s), n0 + 64 * h, k0);
      }
    }
    // Q's four 64-wide K chunks follow the K loop through the ring as if they were iterations
    // nkt .. nkt+3: each lands in the B half of its stage as soon as the last MMA reading that
    // stage has completed, so the load overlaps the tail of the K loop.
    if (ok) {
      mbar_arrive_expect_tx(q_full, STAGES * B_BYTES);
      for (int t = 0; t < STAGES; ++t) {
        const int v = nkt + t;
        const int s = v % STAGES;
        if (!mbar_wait(empty_bar(s), ((uint32_t)(v / STAGES) & 1u) ^ 1u, KID_GEMM_TC, 6)) break;
        const uint32_t sb = smem0 + s * STAGE_BYTES + A_BYTES;
        if (!Q_MN) {
          tma_load_2d(sb, &tmQ, q_full, 64 * t, zq * BN);
        } else {
#pragma unroll
          for (int h = 0; h < BN / 64; ++h) tma_load_2d(sb + h * 8192, &tmQ, q_full, 64 * h, zq * BN + 64 * t);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: the K loop
    for (int i = 0; i < nkt; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      if (!mbar_wait(full_bar(s), ph, KID_GEMM_TC, 7)) break;
      tc_fence_after();
      const uint32_t sa = smem0 + s * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk) {
        const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
        const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
        mma_bf16(tmem_d, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(empty_bar(s));
    }
    mma_commit(accum_bar);
  }
  __syncwarp();

  // ---------------- phase 1: D (TMEM) -> bf16 -> global d1 and the swizzled A tiles in the ring
  bool ok = mbar_wait(accum_bar, 0, KID_GEMM_TC, 8);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  griddep_launch();
  const int r = warp * 32 + lane;  // tile row
  const int m = m0 + r;
  if (ok) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      tmem_wait_ld();
      uint4 q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        q[u] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * u + 0]), __uint_as_float(v[8 * u + 1])),
                          pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                          pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                          pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
      if (args.d1 != nullptr && m < args.M) {
        uint4* g = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(args.d1) + (long)m * args.ld1 + n0 + c);
#pragma unroll
        for (int u = 0; u < 4; ++u) g[u] = q[u];
      }
      // K-major 128-byte swizzle: 16-byte chunk ch of row r sits at chunk position ch ^ (r % 8).
      // K chunk t of D goes to the A half of the stage that holds Q's chunk t.
      uint8_t* tileA = smem + ((nkt + c / 64) % STAGES) * STAGE_BYTES + r * 128;
      const int ch0 = (c % 64) / 8;
#pragma unroll
      for (int u = 0; u < 4; ++u) *reinterpret_cast<uint4*>(tileA + (((ch0 + u) ^ (r & 7)) * 16)) = q[u];
    }
  }
  fence_proxy_async_smem();  // the tensor core reads what the threads just wrote
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---------------- phase 2: out2 = D_tile . Q_block (second accumulator, TMEM columns 256..511)
  if (warp == 1 && lane == 0 && ok) {
    if (mbar_wait(q_full, 0, KID_GEMM_TC, 9)) {
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < STAGES; ++t) {
        const uint32_t sa = smem0 + ((nkt + t) % STAGES) * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < TC_BK / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd = Q_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
          mma_bf16(tmem_d + BN, ad, bd, IDESC2, (t > 0 || kk > 0) ? 1u : 0u);
        }
      }
    }
    mma_commit(acc2_bar);
  }
  __syncwarp();
  bool ok2 = ok && mbar_wait(acc2_bar, 0, KID_GEMM_TC, 10);
  ok2 = __all_sync(0xffffffffu, ok2);
  tc_fence_after();
  if (ok2) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(warp * 32) << 16) + (uint32_t)(BN + c), v);
      tmem_wait_ld();
      float f[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
      if (m < args.M) store32(args.out2, (long)m * args.ld2 + n0 + c, BF16, f);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_d, 2 * BN);
}

// ----------------------------------------- W0' GEMM, 256 x 256 tiles, optional block factor
// One CTA computes a 256 x 256 tile of D = A . B^T (A K-major, B K- or MN-major) as two M = 128
// halves sharing every B tile: per 64-wide k step it issues eight tcgen05.mma (2 halves x 4
// K=16 steps) into two TMEM accumulators (columns 0..255 and 256..511).  Against a 128 x 256
// tile this halves the B bytes per FLOP and doubles the MMA time covered by each ring stage
// (3 stages of 64 KiB), which is what keeps the tensor pipe fed from L2.  With out2 set (b = 256:
// the tile's columns are one block) each half is then written as bf16 into the idle ring in the
// swizzled K-major layout and multiplied by the block's Q (K-major: D . Q^T, forward BD_R;
// MN-major: D . Q, adjoint of BD_P), reusing the half's own TMEM columns once drained.  Q's
// four 64-wide K chunks follow the K loop through the ring (two per stage); the D half uses the
// third stage.  All waits bounded; every thread reaches every barrier.
//
// Q8 (POET-XQ, the replication review of POET-X, "Summary" and "Strengths": the quantised
// variant works through POET-Xmem, so no dequantised weight is ever stored): B is int8 codes
// with one fp32 scale per row of the B array (bscale).  TMA brings each k step's 16 KiB of codes
// into the first half of the stage's B region (so the codes ride the same 3-deep ring as A);
// eight more warps (threads 128..383) read all of them into registers, meet on a named barrier,
// then expand them in place into the stage's swizzled bf16 B tile (scale * code) and signal the
// MMA issuer.
struct WideArgs {
  int M, N, K;
  void* d1;    // bf16 [M, N] store of D (may be null when out2 is set)
  long ld1;
  void* out2;  // bf16 [M, N] block-factor result, or null (plain GEMM)
  long ld2;
  const float* bscale;  // Q8 only: scale of each row of the int8 B array
  int b_early;          // B's first stages are requested before griddep_wait (B is not the previous kernel's output)
};

constexpr int TCW_BM = 256, TCW_BN = 256, TCW_STAGES = 3;
constexpr uint32_t TCW_Q8_TILE = 256 * TC_BK;  // int8 codes of one k step's B tile
constexpr int TCW_CONV_THREADS = 256;           // Q8 converter warps 4..11
constexpr int TCW_CONV_CHUNKS = 2048 / TCW_CONV_THREADS;  // 8-code chunks per converter thread per k step
// Past the ring: the block-factor result's store staging, two 32-row x 64-column boxes per
// epilogue warp, so that it leaves through TMA stores while the ring still holds Q and D.
constexpr uint32_t TCW_OUT_BYTES = 4 * 2 * 4096;
__host__ __device__ constexpr size_t tcw_smem_bytes() {
  return (size_t)TCW_STAGES * (TCW_BM * TC_BK * 2 + TCW_BN * TC_BK * 2) + TCW_OUT_BYTES + 1024 + 256;
}

// Named barrier 1 over the `count` threads of the converter warps, ANDing p across them: every
// participant gets the same answer, so a bounded wait that gave up anywhere ends all of them.
__device__ __forceinline__ bool converters_all(bool p, int count) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, %2, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(count)
      : "memory");
  return r != 0;
}

// Threads of a launch: bf16, 8 warps (warps 0 and 1 also issue the loads and the MMAs; all eight
// drain TMEM, two per lane quarter, each taking half of the columns); Q8, 4 draining warps plus
// the converter warps.
__host__ __device__ constexpr int tcw_threads(bool q8) { return q8 ? 128 + TCW_CONV_THREADS : 256; }

template <bool B_MN, bool Q_MN, bool Q8 = false>
__global__ void __launch_bounds__(tcw_threads(Q8), 1)
    gemm_w256_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmD,
                 const __grid_constant__ CUtensorMap tmO, const WideArgs args) {
  constexpr int BN = TCW_BN, STAGES = TCW_STAGES;
  constexpr uint32_t HALF_A = TC_BM * TC_BK * 2;     // 16 KiB: one 128-row half of an A tile
  constexpr uint32_t A_BYTES = 2 * HALF_A;
  constexpr uint32_t B_BYTES = BN * TC_BK * 2;       // 32 KiB
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t IDESC = sm100::idesc_bf16_f32(TC_BM, BN, false, B_MN);
  constexpr uint32_t IDESC2 = sm100::idesc_bf16_f32(TC_BM, BN, false, Q_MN);
  using namespace sm100;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + TCW_OUT_BYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 3);
  const uint32_t smem0 = smem_u32(smem);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  const uint32_t accum_bar = smem_u32(bars + 2 * STAGES);
  const uint32_t q_full = smem_u32(bars + 2 * STAGES + 1);
  const uint32_t acc2_bar = smem_u32(bars + 2 * STAGES + 2);
  // Q8: B tile of stage s converted (one arrival per converter warp).
  auto conv_bar = [&](int s) { return smem_u32(bars + 2 * STAGES + 4 + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * TCW_BM, n0 = blockIdx.x * BN;
  const int zq = blockIdx.x;
  const int nkt = (args.K + TC_BK - 1) / TC_BK;
  const bool fuse = args.out2 != nullptr;
  // Ring stages used after the K loop: Q chunks 0,1 and 2,3, then the D half.
  const int sq0 = nkt % STAGES, sq1 = (nkt + 1) % STAGES, sdh = (nkt + 2) % STAGES;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accum_bar, 1);
    mbar_init(q_full, 1);
    mbar_init(acc2_bar, 1);
    if (Q8)
      for (int s = 0; s < STAGES; ++s) mbar_init(conv_bar(s), TCW_CONV_THREADS / 32);
    fence_mbar_init();
    fence_proxy_async_smem();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (fuse) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmO);
    }
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_holder;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    // The B tile of step i (W0' or its int8 codes) into the stage's B region.
    auto load_b = [&](int i, int s) {
      const int k0 = i * TC_BK;
      const uint32_t sb = smem0 + s * STAGE_BYTES + A_BYTES;
      if (Q8) {
        if (!B_MN) tma_load_2d(sb, &tmB, full_bar(s), k0, n0);  // box 64 (k) x 256 (n) codes
        else tma_load_2d(sb, &tmB, full_bar(s), n0, k0);        // box 256 (n) x 64 (k) codes
      } else if (!B_MN) {
        tma_load_2d(sb, &tmB, full_bar(s), k0, n0);
      } else {
#pragma unroll
        for (int h = 0; h < BN / 64; ++h) tma_load_2d(sb + h * 8192, &tmB, full_bar(s), n0 + 64 * h, k0);
      }
    };
    const uint32_t stage_tx = Q8 ? A_BYTES + TCW_Q8_TILE : STAGE_BYTES;
    // B of the first stages while the previous kernel (which wrote A) finishes.
    const int early = args.b_early ? min(nkt, STAGES) : 0;
    for (int i = 0; i < early; ++i) {
      mbar_arrive_expect_tx(full_bar(i), stage_tx);
      load_b(i, i);
    }
    griddep_wait();
    bool ok = true;
    for (int i = 0; i < nkt; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      if (i >= early) {
        if (!mbar_wait(empty_bar(s), ph ^ 1u, KID_GEMM_TC, 11)) { ok = false; break; }
        mbar_arrive_expect_tx(full_bar(s), stage_tx);
        load_b(i, s);
      }
      tma_load_2d(smem0 + s * STAGE_BYTES, &tmA, full_bar(s), i * TC_BK, m0);  // box 64 x 256: both halves
    }
    if (ok && fuse) {
      // Q's K chunks t = 0..3 into stages sq0 (t = 0, 1) and sq1 (t = 2, 3), each as soon as the
      // last MMA reading that stage has completed (virtual iterations nkt and nkt + 1).
      mbar_arrive_expect_tx(q_full, 4 * B_BYTES);
      for (int u = 0; u < 2; ++u) {
        const int v = nkt + u;
        const int s = v % STAGES;
        if (!mbar_wait(empty_bar(s), ((uint32_t)(v / STAGES) & 1u) ^ 1u, KID_GEMM_TC, 12)) break;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int t = 2 * u + w;
          const uint32_t dst = smem0 + s * STAGE_BYTES + w * B_BYTES;
          if (!Q_MN) {
            tma_load_2d(dst, &tmQ, q_full, 64 * t, zq * BN);
          } else {
#pragma unroll
            for (int h = 0; h < BN / 64; ++h) tma_load_2d(dst + h * 8192, &tmQ, q_full, 64 * h, zq * BN + 64 * t);
          }
        }
      }
    }
  } else {
    griddep_wait();
  }
  if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: both halves per k step
    for (int i = 0; i < nkt; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      if (!mbar_wait(full_bar(s), ph, KID_GEMM_TC, 13)) break;
      if (Q8 && !mbar_wait(conv_bar(s), ph, KID_GEMM_TC, 19)) break;
      tc_fence_after();
      const uint32_t sa = smem0 + s * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < TC_BK / 16; ++kk) {
        const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
#pragma unroll
        for (int h = 0; h < 2; ++h)
          mma_bf16(tmem_d + h * BN, smem_desc_sw128(sa + h * HALF_A + kk * 32, 16, 1024), bd, IDESC,
                   (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(empty_bar(s));
    }
    mma_commit(accum_bar);
  } else if (Q8 && warp >= 4) {
    // ---------------- converters: codes -> bf16 scale * code in the stage's swizzled B tile.
    // Thread t converts chunks c = CT j + t (CT converter threads, j < 2048 / CT) of 8 codes each.
    // K-major B (rows n, 64 codes each): chunk c is row c / 8, 16-byte chunk c % 8.  MN-major B
    // (rows k, 256 codes each): chunk c is row k = c / 32, columns 8 (c % 32) .. +7, i.e.
    // 64-column sub-tile (c % 32) / 8, chunk c % 8.  Either way the scale belongs to the code's
    // row of B.
    constexpr int CT = TCW_CONV_THREADS, NCH = TCW_CONV_CHUNKS;
    const int t = threadIdx.x - 128;
    float sc[NCH], scn[NCH];
    auto load_scales = [&](int i, float (&dst)[NCH]) {
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int c = j * CT + t;
        const int row = B_MN ? i * TC_BK + (c >> 5) : n0 + (c >> 3);
        dst[j] = row < (B_MN ? args.K : args.N) ? __ldg(args.bscale + row) : 0.f;
      }
    };
    load_scales(0, scn);
    for (int i = 0; i < nkt; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
#pragma unroll
      for (int j = 0; j < NCH; ++j) sc[j] = scn[j];
      if (B_MN && i + 1 < nkt) load_scales(i + 1, scn);  // K-major: the same rows every step
      // All converter warps agree (named barrier) before anyone reads, so a timeout ends all of them.
      if (!converters_all(mbar_wait(full_bar(s), ph, KID_GEMM_TC, 18), CT)) break;
      uint8_t* tile = smem + s * STAGE_BYTES + A_BYTES;
      uint2 code[NCH];
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int c = j * CT + t;
        code[j] = *reinterpret_cast<const uint2*>(tile + (!B_MN ? (c >> 3) * 64 + (c & 7) * 8
                                                                 : (c >> 5) * 256 + (c & 31) * 8));
      }
      converters_all(true, CT);  // every code of the stage is in registers before the expansion
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int c = j * CT + t;
        int dst;
        if (!B_MN) {
          const int row = c >> 3, ch = c & 7;
          dst = row * 128 + ((ch ^ (row & 7)) << 4);
        } else {
          const int row = c >> 5, nc = c & 31;
          dst = (nc >> 3) * 8192 + row * 128 + (((nc & 7) ^ (row & 7)) << 4);
        }
        *reinterpret_cast<uint4*>(tile + dst) = dequant8_bf16(code[j], sc[j]);
      }
      fence_proxy_async_smem();  // the tensor core reads what the threads wrote
      __syncwarp();
      if (lane == 0) mbar_arrive(conv_bar(s));
    }
  }
  __syncwarp();

  bool ok = mbar_wait(accum_bar, 0, KID_GEMM_TC, 14);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  griddep_launch();
  const int lq = warp & 3;                          // TMEM lane quarter of this warp
  const int r = lq * 32 + lane;                     // TMEM lane = row within a half
  const uint32_t tl = tmem_d + ((uint32_t)(lq * 32) << 16);
  const bool epi_warp = !Q8 || warp < 4;            // Q8: the converter warps do not drain
  constexpr int EPI_COLS = Q8 ? BN : BN / 2;        // columns of a 256-column drain per warp
  const int col_lo = Q8 ? 0 : (warp >> 2) * EPI_COLS;

  // Drains this warp's columns of 256 TMEM columns at offset col0 (row m of the output): bf16 to
  // global `dst` (if set) and, if stage >= 0, into that ring stage as four swizzled K-major
  // 128 x 64 tiles, which are both the A operand of the block factor and TMA-store boxes of D.
  auto drain = [&](uint32_t col0, int m, void* dst, long ld, int stage) {
    // 64 columns (two TMEM loads) per round; the next round's loads are in flight while this
    // round's values are converted and written.
    uint32_t va[2][32], vb[2][32];
    tmem_ld_32x32b_x32(tl + col0 + (uint32_t)col_lo, va[0]);
    tmem_ld_32x32b_x32(tl + col0 + (uint32_t)(col_lo + 32), va[1]);
    tmem_wait_ld();
#pragma unroll
    for (int c = col_lo; c < col_lo + EPI_COLS; c += 64) {
      const bool more = c + 64 < col_lo + EPI_COLS;
      if (more) {
        tmem_ld_32x32b_x32(tl + col0 + (uint32_t)(c + 64), vb[0]);
        tmem_ld_32x32b_x32(tl + col0 + (uint32_t)(c + 96), vb[1]);
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t* v = va[hh];
        uint4 q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          q[u] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * u + 0]), __uint_as_float(v[8 * u + 1])),
                            pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                            pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                            pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
        const int cc = c + 32 * hh;
        if (dst != nullptr && m < args.M) {
          uint4* g = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dst) + (long)m * ld + n0 + cc);
#pragma unroll
          for (int u = 0; u < 4; ++u) g[u] = q[u];
        }
        if (stage >= 0) {
          // K chunk cc/64: 16 KiB tile at the stage + (cc/64)*16 KiB, 16-byte chunk ch of row r at
          // chunk position ch ^ (r % 8).
          uint8_t* tileA = smem + stage * STAGE_BYTES + (cc / 64) * HALF_A + r * 128;
          const int ch0 = (cc % 64) / 8;
#pragma unroll
          for (int u = 0; u < 4; ++u) *reinterpret_cast<uint4*>(tileA + (((ch0 + u) ^ (r & 7)) * 16)) = q[u];
        }
      }
      if (more) {
        tmem_wait_ld();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int u = 0; u < 32; ++u) va[hh][u] = vb[hh][u];
      }
    }
  };


  // D goes out through TMA stores of the swizzled tiles (whole 128-byte lines; rows past M are
  // clipped by the tensor map), issued by thread 0 in its bulk group.
  const bool store_d = args.d1 != nullptr;
  auto store_half = [&](int stage, int h) {
    if (threadIdx.x == 0 && store_d) {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        tma_store_2d(&tmD, smem0 + stage * STAGE_BYTES + t * HALF_A, n0 + 64 * t, m0 + h * TC_BM);
      bulk_commit();
    }
  };
  if (!fuse) {
    if (ok && epi_warp) {
      drain(0, m0 + r, nullptr, 0, 0);
      drain(BN, m0 + TC_BM + r, nullptr, 0, 1);
    }
    fence_proxy_async_smem();  // the TMA engine reads what the threads just wrote
    __syncthreads();
    if (ok) {
      store_half(0, 0);
      store_half(1, 1);
    }
  } else {
    // Half h: D_h -> the D stage (bf16, K-major swizzled) -> global d1 by TMA, and the A operand
    // of the block-factor product, whose result lands in the half's own TMEM columns.  The result
    // of half 0 is drained to TMA-store boxes while the product of half 1 runs.
    bool ok2 = ok;
    auto block_product = [&](int h) {
      if (warp == 1 && lane == 0 && ok2) {
        if (mbar_wait(q_full, 0, KID_GEMM_TC, 15)) {
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint32_t sa = smem0 + sdh * STAGE_BYTES + t * HALF_A;
            const uint32_t sb = smem0 + (t < 2 ? sq0 : sq1) * STAGE_BYTES + (t & 1) * B_BYTES;
#pragma unroll
            for (int kk = 0; kk < TC_BK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
              const uint64_t bd = Q_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
              mma_bf16(tmem_d + h * BN, ad, bd, IDESC2, (t > 0 || kk > 0) ? 1u : 0u);
            }
          }
        }
        mma_commit(acc2_bar);
      }
      __syncwarp();
    };
    auto wait_product = [&](int h) {
      if (ok2) ok2 = mbar_wait(acc2_bar, (uint32_t)h, KID_GEMM_TC, 16);
      ok2 = __all_sync(0xffffffffu, ok2);
      tc_fence_after();
    };
    // The block-factor result of half h (TMEM columns col0..): 32-row x 64-column boxes of this
    // warp's columns, stored with TMA (rows past M clipped by the map) from `stage` (nbuf buffers
    // of 4 KiB per warp, used in turn).
    int nbox = 0;
    auto drain_out = [&](uint32_t col0, int h, uint8_t* stage, int nbuf) {
      // One 64-column box per round (two TMEM loads); the next box's loads are in flight while
      // this one is converted, staged and stored.
      const int b0 = col_lo / 64, b1 = (col_lo + EPI_COLS) / 64;
      uint32_t va[2][32], vb[2][32];
      tmem_ld_32x32b_x32(tl + col0 + (uint32_t)(b0 * 64), va[0]);
      tmem_ld_32x32b_x32(tl + col0 + (uint32_t)(b0 * 64 + 32), va[1]);
      tmem_wait_ld();
#pragma unroll
      for (int c64 = b0; c64 < b1; ++c64, ++nbox) {
        const bool more = c64 + 1 < b1;
        if (more) {
          tmem_ld_32x32b_x32(tl + col0 + (uint32_t)(c64 * 64 + 64), vb[0]);
          tmem_ld_32x32b_x32(tl + col0 + (uint32_t)(c64 * 64 + 96), vb[1]);
        }
        uint8_t* buf = stage + (nbox % nbuf) * 4096;
        if (nbox >= nbuf) {
          if (lane == 0) {
            if (nbuf == 1) bulk_wait_read<0>(); else bulk_wait_read<1>();  // this buffer's last store has read it
          }
          __syncwarp();
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t* v = va[hh];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = 8 * u;
            const uint4 q = make_uint4(pack_bf16x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])),
                                       pack_bf16x2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])),
                                       pack_bf16x2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5])),
                                       pack_bf16x2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7])));
            const int ch = hh * 4 + u;
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((ch ^ (lane & 7)) * 16)) = q;
          }
        }
        fence_proxy_async_smem();  // the TMA engine reads what the threads wrote
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmO, smem_u32(buf), n0 + c64 * 64, m0 + h * TC_BM + lq * 32);
          bulk_commit();
        }
        if (more) {
          tmem_wait_ld();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int u = 0; u < 32; ++u) va[hh][u] = vb[hh][u];
        }
      }
    };

    auto stage_d = [&](int h) {
      if (ok2 && epi_warp) drain((uint32_t)(h * BN), m0 + h * TC_BM + r, nullptr, 0, sdh);
      fence_proxy_async_smem();  // the tensor core and the TMA engine read what the threads wrote
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (ok2) store_half(sdh, h);
    };
    // Store staging past the ring: Q8, two 4 KiB buffers for each of the 4 draining warps; bf16,
    // one for each of the 8.
    uint8_t* ostage = smem + STAGES * STAGE_BYTES + (Q8 ? warp * 8192 : warp * 4096);
    stage_d(0);
    block_product(0);
    wait_product(0);
    if (threadIdx.x == 0) bulk_wait_read<0>();  // D_0's stores have read the D stage
    __syncthreads();
    stage_d(1);
    block_product(1);
    if (ok2 && epi_warp) drain_out(0, 0, ostage, Q8 ? 2 : 1);  // beside the second product (other TMEM columns)
    wait_product(1);
    if (Q8) {
      if (ok2 && epi_warp) drain_out(BN, 1, ostage, 2);
    } else {
      // The D stage is free once D_1's stores have read it: two buffers per warp there.
      if (threadIdx.x == 0) bulk_wait_read<0>();
      __syncthreads();
      nbox = 0;  // fresh buffers
      if (ok2) drain_out(BN, 1, smem + sdh * STAGE_BYTES + warp * 8192, 2);
    }
    if (epi_warp && lane == 0) bulk_wait_read<0>();
    __syncwarp();
  }
  // Shared memory stays valid until the stores have read it (the writes complete with the grid).
  if (threadIdx.x == 0) bulk_wait_read<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_d, 2 * BN);
}

// ---------------------------------------------------------------------------- f32 SIMT kernel
struct SimtArgs {
  int M, N, K, splits;
  const float* A;
  long lda, a_zrow, a_zcol;
  int a_mn;
  const float* B;
  long ldb, b_zrow, b_zcol;
  int b_mn;
  Epilogue epi;
};

// 64x64 output tile per 256-thread block, 4x4 per thread, k-steps of 16 staged in smem.
__global__ void __launch_bounds__(256) gemm_f32_simt(const SimtArgs p) {
  sm100::griddep_wait();
  __shared__ float As[16][65];
  __shared__ float Bs[16][65];
  const int z = blockIdx.z / p.splits, split = blockIdx.z % p.splits;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int KT = (p.K + 15) / 16;
  const int kt0 = (int)((long)KT * split / p.splits), kt1 = (int)((long)KT * (split + 1) / p.splits);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int kt = kt0; kt < kt1; ++kt) {
    const int k0 = kt * 16;
    for (int e = threadIdx.x; e < 1024; e += 256) {
      int mm, kk;
      if (p.a_mn) { mm = e & 63; kk = e >> 6; } else { kk = e & 15; mm = e >> 4; }
      const int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < p.M && k < p.K)
        v = p.a_mn ? p.A[((long)z * p.a_zrow + k) * p.lda + (long)z * p.a_zcol + m]
                   : p.A[((long)z * p.a_zrow + m) * p.lda + (long)z * p.a_zcol + k];
      As[kk][mm] = v;
      int nn, kb;
      if (p.b_mn) { nn = e & 63; kb = e >> 6; } else { kb = e & 15; nn = e >> 4; }
      const int n = n0 + nn, kq = k0 + kb;
      float w = 0.f;
      if (n < p.N && kq < p.K)
        w = p.b_mn ? p.B[((long)z * p.b_zrow + kq) * p.ldb + (long)z * p.b_zcol + n]
                   : p.B[((long)z * p.b_zrow + n) * p.ldb + (long)z * p.b_zcol + kq];
      Bs[kb][nn] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < p.M && n < p.N) epilogue1(p.epi, z, split, m, n, acc[i][j]);
    }
}

}  // namespace poetx
