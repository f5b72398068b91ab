// Fused Cayley–Neumann kernels: the whole CNP forward (or its adjoint) of every block in one
// launch (replication review of POET-X, "Summary": a fused kernel for the Cayley–Neumann
// series that reuses the lower powers; "Reproducibility & code": forward and grad-Q kernels).
//
// Each b x b block (b <= 256) is owned by one thread-block cluster of (b/BN) x ceil(b/128) CTAs;
// CTA (n-tile, m-tile) owns the same 128 x BN tile of every intermediate of its block.  The
// kernel runs a short program of stages:
//   GEMM stage  — tile of D = A . B^T on tcgen05 (A: S or the stacked adjoint terms, K-major;
//                 B: the previous power / adjoint term, streamed from L2 by TMA);
//   UNPACK      — packed theta -> S;
//   REDUCE      — split-K partial sum of G = dL/dQ, fused with UNPACK;
//   PACK        — g[p(i,j)] = G_S[i][j] - G_S[j][i].
// Per-row state that only the owning CTA reads back (S, T = S + M_k, G, the running sum E)
// stays in TMEM beside the accumulator: four regions of BN fp32 columns (ACC, R1, R2, R3), one
// TMEM lane per tile row, read and written by the thread that owns the row.  Only operands
// that peer CTAs consume (bf16 S, M_j, adjoint terms), the f32 G_S needed by PACK and the final
// outputs go through global memory.  Between stages each CTA publishes its tile (stores, proxy
// fence for the peers' TMA reads) and meets the others at a cluster barrier; every CTA executes
// every barrier of the program, whatever happens to its bounded waits.
#pragma once

#include "common.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "sm100.cuh"

namespace poetx {

constexpr int CNP_MAX_STAGES = 20;
constexpr int CNP_THREADS = 256;  // 8 warps: warp w owns TMEM lane quarter w%4, column half w/4
enum CnpStageKind : int { CNP_GEMM = 0, CNP_UNPACK = 1, CNP_REDUCE_UNPACK = 2, CNP_PACK = 3 };
enum CnpReg : int { CNP_NONE = -1, CNP_ACC = 0, CNP_R1 = 1, CNP_R2 = 2, CNP_R3 = 3 };
enum : int { KID_CNP_FUSED = 2 };

// Stage description shared by the segments (register-form epilogue):
//   out1 = alpha1*acc + beta1*REG[c_reg] (+ I if diag1)  -> global g1 (g1_dtype) and/or REG[r1]
//   out2 = alpha2*acc + beta2*REG[c_reg] (+ REG[r2] if accum2) -> REG[r2]
struct CnpStageDesc {
  int kind;
  int b_mn;
  int c_reg;
  float alpha1, beta1;
  int diag1;
  int r1;
  int g1_dtype;  // BF16 or F32 (g1 may be null per segment)
  int r2;
  float alpha2, beta2;
  int accum2;
};

struct CnpSegStage {
  CUtensorMap tmA;  // K-major A operand map (box 64 x 128)
  CUtensorMap tmB;  // B operand map (K-major box 64 x BN, or MN-major box 64 x 64)
  CUtensorMap tmD;  // store map of g1 (128-byte x 32-row boxes: 64 bf16 or 32 fp32 columns)
  int K;
  int a_zrow, b_zrow, b_zcol;
  void* g1;         // global out1: element (z*b+i, j) at g1[(z*b+i)*g1_ld + j]
  long g1_ld;
};

struct CnpSegment {
  int nb;
  const float* theta;  // [nb, b(b-1)/2]
  // UNPACK: S -> R1 (unless no_sreg), two optional bf16 global copies, optional identity.
  int no_sreg;
  void* Sb0;
  long ld0;
  void* Sb1;
  long ld1;
  int add_identity;
  // REDUCE: G = sum of split-K partials -> R2, optional bf16 copy Gb, optional f32 copy G32.
  const float* part;  // [splits][nb*b][b]
  int splits;
  void* Gb;
  long ldg;
  float* G32;
  // PACK
  const float* GS;    // [nb*b][b] f32
  float* grad;        // [nb, b(b-1)/2]
};

struct CnpProgram {
  int b;
  int nstages;
  int nseg;
  CnpStageDesc st[CNP_MAX_STAGES];
  CnpSegment seg[2];
  CnpSegStage g[CNP_MAX_STAGES][2];
};

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Shared memory of the program kernel: the TMA ring, or two padded 128 x BN f32 staging tiles
// (whichever is larger), then the barriers.
template <int BN, int STAGES>
__host__ __device__ constexpr size_t cnp_data_bytes() {
  return (size_t)STAGES * (TC_BM * TC_BK * 2 + BN * TC_BK * 2) > (size_t)2 * TC_BM * (BN + 4) * 4
             ? (size_t)STAGES * (TC_BM * TC_BK * 2 + BN * TC_BK * 2)
             : ((size_t)2 * TC_BM * (BN + 4) * 4 + 1023) / 1024 * 1024;
}
template <int BN, int STAGES>
__host__ __device__ constexpr size_t cnp_smem_bytes() {
  return cnp_data_bytes<BN, STAGES>() + 1024 /*align*/ + 256 /*barriers*/;
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(CNP_THREADS, 1) cnp_program_kernel(const __grid_constant__ CnpProgram prog) {
  constexpr uint32_t A_BYTES = TC_BM * TC_BK * 2;
  constexpr uint32_t B_BYTES = BN * TC_BK * 2;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = 4 * BN;  // ACC, R1, R2, R3
  constexpr int HALF = BN / 2;            // columns per warp (two warps share a lane quarter)
  static_assert(HALF % 32 == 0, "tile half must be whole 32-column chunks");
  using namespace sm100;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + cnp_data_bytes<BN, STAGES>());
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  const uint32_t smem0 = smem_u32(smem);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  const uint32_t accum_bar = smem_u32(bars + 2 * STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int b = prog.b;
  const int zg = blockIdx.z;
  const int seg = (prog.nseg > 1 && zg >= prog.seg[0].nb) ? 1 : 0;
  const int z = seg ? zg - prog.seg[0].nb : zg;
  const CnpSegment& S = prog.seg[seg];
  const int m0 = blockIdx.y * TC_BM, n0 = blockIdx.x * BN;
  const long P = (long)b * (b - 1) / 2;
  const float* th = S.theta + (long)z * P;
  const int i = m0 + quarter * 32 + lane;  // the tile row this thread owns
  const bool row_ok = i < b;
  const long grow = (long)z * b + i;       // row in the [nb*b, *] scratch arrays

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accum_bar, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem0 = *tmem_holder;
  const uint32_t tlane = tmem0 + ((uint32_t)(quarter * 32) << 16);
  auto treg = [&](int reg, int col) { return tlane + (uint32_t)(reg * BN + col); };
  // Two 128 x BN f32 staging tiles (padded row stride), overlaid on the TMA ring, which is idle
  // whenever they are in use (between the last MMA of a stage and the first TMA load of the next).
  constexpr int TS = BN + 4;  // padded row stride (16-byte aligned rows for float4 access)
  float* T0 = reinterpret_cast<float*>(smem);
  float* T1 = T0 + TC_BM * TS;
  // Coalesced write of a staged tile to global: warps over rows, lanes along columns.  With
  // `skew` the tile holds theta unsigned and entries below the diagonal are negated on the way.
  auto tile_store = [&](const float* T, void* dst, long ld, int dt, bool skew) {
    for (int r = warp; r < TC_BM; r += CNP_THREADS / 32) {
      const int ii = m0 + r;
      if (ii >= b) break;
      const long base = ((long)z * b + ii) * ld + n0;
      for (int cc = lane * 4; cc < BN; cc += 128) {
        float4 f = *reinterpret_cast<const float4*>(T + r * TS + cc);
        if (skew) {
          const int jj = n0 + cc;
          if (jj < ii) f.x = -f.x;
          if (jj + 1 < ii) f.y = -f.y;
          if (jj + 2 < ii) f.z = -f.z;
          if (jj + 3 < ii) f.w = -f.w;
        }
        if (dt == BF16) {
          uint2 u;
          u.x = pack_bf16x2(f.x, f.y);
          u.y = pack_bf16x2(f.z, f.w);
          *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(dst) + base + cc) = u;
        } else {
          *reinterpret_cast<float4*>(reinterpret_cast<float*>(dst) + base + cc) = f;
        }
      }
    }
  };
  uint32_t it = 0;
  uint32_t acc_phase = 0;

  for (int s = 0; s < prog.nstages; ++s) {
    const CnpStageDesc& D = prog.st[s];
    bool wrote_global = false, wrote_tmem = false;
    if (D.kind == CNP_GEMM) {
      const CnpSegStage& G = prog.g[s][seg];
      const bool b_mn = D.b_mn != 0;
      const int nkt = (G.K + TC_BK - 1) / TC_BK;
      const uint32_t idesc = idesc_bf16_f32(TC_BM, BN, false, b_mn);
      if (warp == 0 && lane == 0) {
        for (int k = 0; k < nkt; ++k) {
          const uint32_t q = it + k;
          const int stg = q % STAGES;
          const uint32_t ph = (q / STAGES) & 1u;
          if (!mbar_wait(empty_bar(stg), ph ^ 1u, KID_CNP_FUSED, 1)) break;
          mbar_arrive_expect_tx(full_bar(stg), STAGE_BYTES);
          const int k0 = k * TC_BK;
          const uint32_t sa = smem0 + stg * STAGE_BYTES, sb = sa + A_BYTES;
          tma_load_2d(sa, &G.tmA, full_bar(stg), k0, z * G.a_zrow + m0);
          if (!b_mn) {
            tma_load_2d(sb, &G.tmB, full_bar(stg), z * G.b_zcol + k0, z * G.b_zrow + n0);
          } else {
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_2d(sb + h * 8192, &G.tmB, full_bar(stg), z * G.b_zcol + n0 + 64 * h, z * G.b_zrow + k0);
          }
        }
      } else if (warp == 1 && lane == 0) {
        for (int k = 0; k < nkt; ++k) {
          const uint32_t q = it + k;
          const int stg = q % STAGES;
          const uint32_t ph = (q / STAGES) & 1u;
          if (!mbar_wait(full_bar(stg), ph, KID_CNP_FUSED, 2)) break;
          tc_fence_after();
          const uint32_t sa = smem0 + stg * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = b_mn ? smem_desc_sw128(sb + kk * 2048, 8192, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
            mma_bf16(tmem0, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(empty_bar(stg));
        }
        mma_commit(accum_bar);
      }
      __syncwarp();
      it += nkt;
      bool ok = mbar_wait(accum_bar, acc_phase, KID_CNP_FUSED, 3);
      acc_phase ^= 1u;
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      // Staging of this warp's 32 x HALF slice of out1 for the TMA store: 128-byte rows,
      // 16-byte chunk ch of row `lane` at position ch ^ (lane % 8), one 4 KiB box per 128 bytes
      // of row (the ring is idle: every MMA of the stage has completed).
      const bool f32_out = D.g1_dtype == F32;
      uint8_t* stg = smem + warp * 8192;
      const bool rows_ok = m0 + quarter * 32 < b;  // b % 32 == 0: a 32-row box is all in or all out
      // A bf16 box is 64 columns wide: with BN = 64 a warp's slice is narrower, so those tiles
      // keep per-row stores.
      const bool tma_out = G.g1 != nullptr && (f32_out ? HALF % 32 : HALF % 64) == 0;
      if (ok) {
#pragma unroll 1
        for (int c = half * HALF; c < (half + 1) * HALF; c += 32) {
          uint32_t ra[32], rc[32], re[32];
          tmem_ld_32x32b_x32(treg(CNP_ACC, c), ra);
          if (D.c_reg >= 0) tmem_ld_32x32b_x32(treg(D.c_reg, c), rc);
          if (D.r2 >= 0 && D.accum2) tmem_ld_32x32b_x32(treg(D.r2, c), re);
          tmem_wait_ld();
          const int n = n0 + c;
          if (D.r2 >= 0) {  // out2 first, in place in re (it needs acc and the addend only)
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float v = D.alpha2 * __uint_as_float(ra[j]);
              if (D.c_reg >= 0) v += D.beta2 * __uint_as_float(rc[j]);
              if (D.accum2) v += __uint_as_float(re[j]);
              re[j] = __float_as_uint(v);
            }
            tmem_st_32x32b_x32(treg(D.r2, c), re);
            wrote_tmem = true;
          }
          float o1[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float v = D.alpha1 * __uint_as_float(ra[j]);
            if (D.c_reg >= 0) v += D.beta1 * __uint_as_float(rc[j]);
            if (D.diag1 && i == n + j) v += 1.f;
            o1[j] = v;
          }
          if (D.r1 >= 0) {
            tmem_st_32x32b_x32(treg(D.r1, c), reinterpret_cast<const uint32_t (&)[32]>(o1));
            wrote_tmem = true;
          }
          if (G.g1 != nullptr && !tma_out && row_ok) {
            store32(G.g1, grow * G.g1_ld + n, D.g1_dtype, o1);
            wrote_global = true;
          } else if (tma_out) {
            const int cl = c - half * HALF;  // column of this chunk within the warp's slice
            if (f32_out) {
              uint8_t* box = stg + (cl / 32) * 4096 + lane * 128;
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<float4*>(box + ((u ^ (lane & 7)) * 16)) =
                    make_float4(o1[4 * u], o1[4 * u + 1], o1[4 * u + 2], o1[4 * u + 3]);
            } else {
              uint8_t* box = stg + (cl / 64) * 4096 + lane * 128;
              const int ch0 = (cl % 64) / 8;
#pragma unroll
              for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4*>(box + (((ch0 + u) ^ (lane & 7)) * 16)) =
                    make_uint4(pack_bf16x2(o1[8 * u], o1[8 * u + 1]), pack_bf16x2(o1[8 * u + 2], o1[8 * u + 3]),
                               pack_bf16x2(o1[8 * u + 4], o1[8 * u + 5]), pack_bf16x2(o1[8 * u + 6], o1[8 * u + 7]));
            }
          }
        }
      }
      if (tma_out) {
        // One lane stores the warp's boxes; the stores are complete (visible to the peers' TMA
        // loads of the next stage after the cluster barrier) before the barrier.
        wrote_global = true;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok && rows_ok) {
          const int x0 = n0 + half * HALF, y0 = z * b + m0 + quarter * 32;
          const int nbox = f32_out ? HALF / 32 : HALF / 64;
          for (int t = 0; t < nbox; ++t)
            tma_store_2d(&G.tmD, smem_u32(stg + t * 4096), x0 + t * (f32_out ? 32 : 64), y0);
          bulk_commit();
          bulk_wait<0>();
        }
        __syncwarp();
      }
    } else if (D.kind == CNP_UNPACK || D.kind == CNP_REDUCE_UNPACK) {
      // theta -> T0 by per-thread asynchronous copies (all of a thread's copies in flight at
      // once, no registers held): above the diagonal warps walk rows (theta's packed row i is
      // contiguous in j), below it warps walk columns (packed row j is contiguous in i).  T0
      // holds theta unsigned; the consumers negate below the diagonal.  Packed row i starts at
      // ro(i) + i + 1 with ro(i) = i*b - i(i+1)/2 - i - 1, so element (i, j) is ro(i) + j.
      constexpr int RW = TC_BM / (CNP_THREADS / 32);  // rows (or columns) per warp
      constexpr int CPL = BN / 32;                    // columns (or rows / 32) per lane
      constexpr int RPL = TC_BM / 32;                 // rows per lane in the column walk
      const float diag = S.add_identity ? 1.f : 0.f;
#pragma unroll 4
      for (int t = 0; t < RW; ++t) {
        const int r = warp + 8 * t, ii = m0 + r;
        const int ro = ii * b - (ii * (ii + 1)) / 2 - ii - 1;
#pragma unroll
        for (int q = 0; q < CPL; ++q) {
          const int cc = lane + 32 * q, jj = n0 + cc;
          float* dst = T0 + r * TS + cc;
          if (jj > ii) {
            if (ii < b) cp_async4(dst, th + (ro + jj));
            else *dst = 0.f;
          } else if (jj == ii) {
            *dst = diag;
          }
        }
      }
#pragma unroll 4
      for (int t = 0; t < BN / 8; ++t) {
        const int cc = warp + 8 * t, jj = n0 + cc;
        const int ro = jj * b - (jj * (jj + 1)) / 2 - jj - 1;
#pragma unroll
        for (int q = 0; q < RPL; ++q) {
          const int r = lane + 32 * q, ii = m0 + r;
          if (ii > jj) {
            float* dst = T0 + r * TS + cc;
            if (ii < b) cp_async4(dst, th + (ro + ii));
            else *dst = 0.f;
          }
        }
      }
      if (D.kind == CNP_REDUCE_UNPACK && S.splits == 1) {
        // G (one partial: the gradient GEMM did not split K) -> T1, 16-byte copies by rows.
        if (lane * 4 < BN) {
#pragma unroll 4
          for (int t = 0; t < RW; ++t) {
            const int ii = m0 + warp + 8 * t;
            float* dst = T1 + (warp + 8 * t) * TS + lane * 4;
            if (ii < b) cp_async16(dst, S.part + ((long)z * b + ii) * b + n0 + lane * 4);
            else *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
      cp_async_wait_all();
      if (D.kind == CNP_REDUCE_UNPACK && S.splits > 1) {
        // G = sum of split-K partials -> T1, row walk with one float4 per lane per row.
        const long sstride = (long)S.nb * b * b;
        constexpr int RB = 4;
#pragma unroll 1
        for (int t0 = 0; t0 < RW; t0 += RB) {
          float4 acc4[RB];
#pragma unroll
          for (int t = 0; t < RB; ++t) acc4[t] = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int sp0 = 0; sp0 < S.splits; sp0 += 4) {  // four splits' loads in flight at once
            float4 ld4[4][RB];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
              for (int t = 0; t < RB; ++t) {
                const int ii = m0 + warp + 8 * (t0 + t), sp = sp0 + u;
                ld4[u][t] = (sp < S.splits && ii < b && lane * 4 < BN)
                                ? __ldg(reinterpret_cast<const float4*>(S.part + sp * sstride + ((long)z * b + ii) * b + n0) + lane)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
              for (int t = 0; t < RB; ++t) {
                acc4[t].x += ld4[u][t].x; acc4[t].y += ld4[u][t].y; acc4[t].z += ld4[u][t].z; acc4[t].w += ld4[u][t].w;
              }
          }
#pragma unroll
          for (int t = 0; t < RB; ++t)
            if (lane * 4 < BN) *reinterpret_cast<float4*>(T1 + (warp + 8 * (t0 + t)) * TS + lane * 4) = acc4[t];
        }
      }
      __syncthreads();
      // Coalesced global copies from the tiles; then each thread moves its row into TMEM.
      if (S.Sb0) tile_store(T0, S.Sb0, S.ld0, BF16, true);
      if (S.Sb1) tile_store(T0, S.Sb1, S.ld1, BF16, true);
      if (D.kind == CNP_REDUCE_UNPACK) {
        if (S.Gb) tile_store(T1, S.Gb, S.ldg, BF16, false);
        if (S.G32) tile_store(T1, S.G32, b, F32, false);
      }
      wrote_global = true;
#pragma unroll 1
      for (int c = half * HALF; c < (half + 1) * HALF; c += 32) {
        uint32_t w[32];
        if (!S.no_sreg) {
          const float4* trow = reinterpret_cast<const float4*>(T0 + (quarter * 32 + lane) * TS + c);
          const int neg_below = i - (n0 + c);  // columns j < neg_below of this chunk lie below the diagonal
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 f = trow[j];
            w[4 * j] = __float_as_uint(4 * j < neg_below ? -f.x : f.x);
            w[4 * j + 1] = __float_as_uint(4 * j + 1 < neg_below ? -f.y : f.y);
            w[4 * j + 2] = __float_as_uint(4 * j + 2 < neg_below ? -f.z : f.z);
            w[4 * j + 3] = __float_as_uint(4 * j + 3 < neg_below ? -f.w : f.w);
          }
          tmem_st_32x32b_x32(treg(CNP_R1, c), w);
          wrote_tmem = true;
        }
        if (D.kind == CNP_REDUCE_UNPACK) {
          const float4* grow4 = reinterpret_cast<const float4*>(T1 + (quarter * 32 + lane) * TS + c);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 f = grow4[j];
            w[4 * j] = __float_as_uint(f.x); w[4 * j + 1] = __float_as_uint(f.y);
            w[4 * j + 2] = __float_as_uint(f.z); w[4 * j + 3] = __float_as_uint(f.w);
          }
          tmem_st_32x32b_x32(treg(CNP_R2, c), w);
          wrote_tmem = true;
        }
      }
    } else if (D.kind == CNP_PACK) {
      // T0 = own tile of G_S (16-byte copies by rows), T1[i][j] = G_S[j][i] (4-byte copies,
      // column walk, contiguous in i); then g[p(i,j)] = T0 - T1 with lanes along j (contiguous
      // in p).  All copies of a thread are in flight at once.
      constexpr int RW = TC_BM / (CNP_THREADS / 32);
      constexpr int RPL = TC_BM / 32;
      if (lane * 4 < BN) {
#pragma unroll 4
        for (int t = 0; t < RW; ++t) {
          const int ii = m0 + warp + 8 * t;
          if (ii < b) cp_async16(T0 + (warp + 8 * t) * TS + lane * 4, S.GS + ((long)z * b + ii) * b + n0 + lane * 4);
        }
      }
#pragma unroll 4
      for (int t = 0; t < BN / 8; ++t)
#pragma unroll
        for (int q = 0; q < RPL; ++q) {
          const int jj = n0 + warp + 8 * t, ii = m0 + lane + 32 * q;
          if (ii < b) cp_async4(T1 + (lane + 32 * q) * TS + warp + 8 * t, S.GS + ((long)z * b + jj) * b + ii);
        }
      cp_async_wait_all();
      __syncthreads();
      for (int r = warp; r < TC_BM; r += CNP_THREADS / 32) {
        const int ii = m0 + r;
        if (ii >= b) break;
        for (int cc = lane; cc < BN; cc += 32) {
          const int jj = n0 + cc;
          if (ii < jj) S.grad[(long)z * P + packed_pos(ii, jj, b)] = T0[r * TS + cc] - T1[r * TS + cc];
        }
      }
    }
    if (wrote_tmem) tmem_wait_st();
    if (wrote_global) fence_proxy_async_global();
    tc_fence_before();
    cluster_sync_all();
    fence_proxy_async_global();  // the next stage's TMA reads see the peers' generic-proxy writes
    tc_fence_after();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem0, TMEM_COLS);
}

}  // namespace poetx
