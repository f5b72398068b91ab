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
  CUtensorMap tmS0, tmS1;  // store maps of Sb0 / Sb1 (bf16, 64-column x 32-row boxes)
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

// Shared memory of the program kernel: the TMA ring of the GEMM stages, overlaid by the staging
// of the elementwise stages (UNPACK: theta row segments above the diagonal, 128 x (BN + 8) f32,
// and column segments below it, BN x 136 f32, plus the G tile, 128 x (BN + 4) f32; PACK: the
// own G_S tile and the rows of the mirrored one, 128 x (BN + 4) and BN x 132 f32), then the
// barriers.
// UNPACK staging: the theta segments of a tile (at most 128 x BN elements in all, plus 11
// floats of alignment slack per segment), 8 warps x 4 KiB of bf16 boxes for the TMA store of S,
// the G tile (pitch BN + 4) and the segment offsets.
template <int BN>
__host__ __device__ constexpr size_t cnp_stage_bytes() {
  return (((size_t)TC_BM * BN + 11 * (size_t)(TC_BM + BN)) * 4 + 1023) / 1024 * 1024;
}
template <int BN>
__host__ __device__ constexpr size_t cnp_ew_bytes() {
  return cnp_stage_bytes<BN>() + 8 * 4096 + (size_t)TC_BM * (BN + 4) * 4 + 4096;
}
template <int BN, int STAGES>
__host__ __device__ constexpr size_t cnp_data_bytes() {
  return ((size_t)STAGES * (TC_BM * TC_BK * 2 + BN * TC_BK * 2) > cnp_ew_bytes<BN>()
              ? (size_t)STAGES * (TC_BM * TC_BK * 2 + BN * TC_BK * 2)
              : cnp_ew_bytes<BN>() + 1023) / 1024 * 1024;
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
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 2);
  const uint32_t smem0 = smem_u32(smem);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  const uint32_t accum_bar = smem_u32(bars + 2 * STAGES);
  const uint32_t ew_bar = smem_u32(bars + 2 * STAGES + 1);  // bulk copies of an elementwise stage

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
    mbar_init(ew_bar, CNP_THREADS);
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
  griddep_wait();  // theta and the gradient partials come from earlier kernels
  auto treg = [&](int reg, int col) { return tlane + (uint32_t)(reg * BN + col); };
  // The elementwise stages stage their tiles in the TMA ring, which is idle whenever they run
  // (between the last MMA of a stage and the first TMA load of the next).
  constexpr int TS = BN + 4;  // padded row stride of a staged f32 tile (16-byte aligned rows)
  // Coalesced write of a staged f32 tile (row pitch `pitch` floats) to global: warps over rows,
  // lanes along columns, four columns per lane.
  auto tile_store = [&](const float* T, int pitch, void* dst, long ld, int dt) {
    for (int r = warp; r < TC_BM; r += CNP_THREADS / 32) {
      const int ii = m0 + r;
      if (ii >= b) break;
      const long base = ((long)z * b + ii) * ld + n0;
      for (int cc = lane * 4; cc < BN; cc += 128) {
        const float* src = T + r * pitch + cc;
        const float4 f = make_float4(src[0], src[1], src[2], src[3]);
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
  uint32_t ew_phase = 0;
  // One 1-D bulk copy per thread (or none) of `bytes` from global `src` to shared `dst`, counted
  // on ew_bar; every thread arrives exactly once.
  auto bulk_one = [&](void* dst, const void* src, uint32_t bytes) {
    if (bytes > 0) {
      fence_proxy_async_smem();  // the copy overwrites what earlier stages wrote and read
      mbar_arrive_expect_tx(ew_bar, bytes);
      bulk_load_1d(smem_u32(dst), src, bytes, ew_bar);
    } else {
      mbar_arrive(ew_bar);
    }
  };

  for (int s = 0; s < prog.nstages; ++s) {
    const CnpStageDesc& D = prog.st[s];
    if (s == prog.nstages - 1) griddep_launch();
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
      // theta -> S.  Above the diagonal the tile row r (i = m0 + r) needs the segment
      // j = max(n0, i+1) .. n0+BN-1 of packed row i; below it tile column cc (j = n0 + cc) needs
      // the segment i = max(m0, j+1) .. min(m0+128, b)-1 of packed row j (S[i][j] = -theta[p(j,i)]).
      // Each segment is one 1-D bulk copy of its 16-byte-aligned cover into a compact staging
      // area (thread t < 128: row t; 128 <= t < 128 + BN: column t - 128; element e of a
      // segment starting at packed offset e0 sits at e0 % 4 + e of its slot), then the tile is
      // assembled in T0 (pitch BN + 1): rows with lanes along j, columns with lanes along i,
      // both conflict-free.  Packed row i starts at ro(i) + i + 1, ro(i) = i*b - i(i+1)/2 - i - 1.
      constexpr int RW = TC_BM / (CNP_THREADS / 32);
      float* Sg = reinterpret_cast<float*>(smem);
      uint8_t* stg = smem + cnp_stage_bytes<BN>() + warp * 4096;  // this warp's bf16 box
      float* Gt = reinterpret_cast<float*>(smem + cnp_stage_bytes<BN>() + 8 * 4096);  // G tile, pitch TS
      int* seg_off = reinterpret_cast<int*>(Gt + TC_BM * TS);  // [256]: slot start + e0 % 4
      int* colbase = seg_off + CNP_THREADS + 8;               // [BN]: Sg index of row 0 of column cc
      auto ro = [&](int r) { return r * b - (r * (r + 1)) / 2 - r - 1; };
      auto seg_of = [&](int t, int& e0, int& cnt) {  // segment of thread t's row / column
        e0 = 0; cnt = 0;
        if (t < TC_BM) {
          const int ii = m0 + t, jlo = max(n0, ii + 1);
          if (ii < b && jlo < n0 + BN) { e0 = ro(ii) + jlo; cnt = n0 + BN - jlo; }
        } else if (t < TC_BM + BN) {
          const int jj = n0 + t - TC_BM, ilo = max(m0, jj + 1), ihi = min(m0 + TC_BM, b);
          if (ilo < ihi) { e0 = ro(jj) + ilo; cnt = ihi - ilo; }
        }
      };
      {
        const int t = threadIdx.x;
        int e0, cnt;
        seg_of(t, e0, cnt);
        // slot start: exclusive prefix sum over threads of len + 11 floats rounded up to 4
        const int cap = cnt > 0 ? (cnt + 11) & ~3 : 0;
        int x = cap;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, d);
          if (lane >= d) x += y;
        }
        int* warp_sum = seg_off + CNP_THREADS;
        if (lane == 31) warp_sum[warp] = x;
        __syncthreads();
        int off = x - cap;
        for (int w = 0; w < warp; ++w) off += warp_sum[w];
        seg_off[t] = off + (e0 & 3);
        if (t >= TC_BM && t < TC_BM + BN) colbase[t - TC_BM] = off + (e0 & 3) - (max(m0, n0 + t - TC_BM + 1) - m0);
        // block z's theta starts 16-byte aligned (P * 4 is a multiple of 16 for b % 8 == 0), so
        // the rounded cover never leaves it
        const int b0 = (e0 * 4) & ~15, b1 = ((e0 + cnt) * 4 + 15) & ~15;
        bulk_one(Sg + off, reinterpret_cast<const char*>(th) + b0, cnt > 0 ? (uint32_t)(b1 - b0) : 0u);
      }
      if (D.kind == CNP_REDUCE_UNPACK && S.splits == 1) {
        // G (one partial: the gradient GEMM did not split K) -> Gt, 16-byte copies by rows.
        if (lane * 4 < BN) {
#pragma unroll 4
          for (int t = 0; t < RW; ++t) {
            const int ii = m0 + warp + 8 * t;
            float* dst = Gt + (warp + 8 * t) * TS + lane * 4;
            if (ii < b) cp_async16(dst, S.part + ((long)z * b + ii) * b + n0 + lane * 4);
            else *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
      if (D.kind == CNP_REDUCE_UNPACK && S.splits > 1) {
        // G = sum of split-K partials -> Gt, row walk with one float4 per lane per row.
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
            if (lane * 4 < BN) *reinterpret_cast<float4*>(Gt + (warp + 8 * (t0 + t)) * TS + lane * 4) = acc4[t];
        }
      }
      cp_async_wait_all();
      bool got = mbar_wait(ew_bar, ew_phase, KID_CNP_FUSED, 4);
      ew_phase ^= 1u;
      got = __syncthreads_and(got);
      // Each thread builds its tile row (r = 32 quarter + lane) over its half of the columns
      // straight from the staging: above the diagonal from the row's own segment, below it from
      // the column segments (lanes read consecutive rows of one segment); S goes to TMEM (R1)
      // and, as bf16, through a swizzled 32 x 64 box and a TMA store to Sb0 / Sb1.
      const float diag = S.add_identity ? 1.f : 0.f;
      const int r_own = quarter * 32 + lane, i_own = m0 + r_own;
      const int ld_c = i_own - n0;  // this row's diagonal column
      const int rowbase = seg_off[r_own] - (max(n0, i_own + 1) - n0);
      const bool s_out = S.Sb0 != nullptr || S.Sb1 != nullptr;
      const bool s_tma = HALF % 64 == 0;  // a bf16 box is 64 columns wide
      const bool rows_ok = m0 + quarter * 32 < b;
      if (D.kind == CNP_REDUCE_UNPACK) {
        if (S.Gb) tile_store(Gt, TS, S.Gb, S.ldg, BF16);
        if (S.G32) tile_store(Gt, TS, S.G32, b, F32);
      }
      wrote_global = true;
#pragma unroll 1
      for (int c = half * HALF; c < (half + 1) * HALF; c += 32) {
        uint32_t w[32];
        float v[32];
        // One unconditional shared load per element (its address selected; element 0 of the
        // staging where nothing is read: dead rows and the diagonal), so the 32 loads of a chunk
        // are independent and pipeline.
        const bool live = i_own < b && got;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int cc = c + j;
          const bool up = cc > ld_c;
          const int idx = (!live || cc == ld_c) ? 0 : (up ? rowbase + cc : colbase[cc] + r_own);
          const float x = Sg[idx];
          v[j] = !live ? 0.f : (up ? x : (cc == ld_c ? diag : -x));
          w[j] = __float_as_uint(v[j]);
        }
        if (!S.no_sreg) {
          tmem_st_32x32b_x32(treg(CNP_R1, c), w);
          wrote_tmem = true;
        }
        if (s_out) {
          if (s_tma) {
            uint8_t* box = stg + lane * 128;
            const int ch0 = ((c - half * HALF) % 64) / 8;
#pragma unroll
            for (int u = 0; u < 4; ++u)
              *reinterpret_cast<uint4*>(box + (((ch0 + u) ^ (lane & 7)) * 16)) =
                  make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                             pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
          } else if (i_own < b) {
            if (S.Sb0) store32(S.Sb0, ((long)z * b + i_own) * S.ld0 + n0 + c, BF16, v);
            if (S.Sb1) store32(S.Sb1, ((long)z * b + i_own) * S.ld1 + n0 + c, BF16, v);
          }
        }
        if (D.kind == CNP_REDUCE_UNPACK) {
          const float4* grow4 = reinterpret_cast<const float4*>(Gt + (quarter * 32 + lane) * TS + c);
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
      if (s_out && s_tma) {
        // one lane stores the warp's box (complete before the stage barrier: peers read S next)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && got && rows_ok) {
          const int x0 = n0 + half * HALF, y0 = z * b + m0 + quarter * 32;
          if (S.Sb0) tma_store_2d(&S.tmS0, smem_u32(stg), x0, y0);
          if (S.Sb1) tma_store_2d(&S.tmS1, smem_u32(stg), x0, y0);
          bulk_commit();
          bulk_wait<0>();
        }
        __syncwarp();
      }
    } else if (D.kind == CNP_PACK) {
      // Own tile of G_S -> Tp (rows, pitch TS) and rows n0.. of G_S restricted to columns m0..
      // -> Tt (row cc holds G_S[n0+cc][m0 + r], pitch 132): one 1-D bulk copy per row (thread
      // t < 128: own row t; 128 <= t < 128 + BN: mirrored row t - 128).  Then
      // g[p(i,j)] = G_S[i][j] - G_S[j][i] with lanes along j (contiguous in p).
      constexpr int TP = TC_BM + 4;
      float* Tp = reinterpret_cast<float*>(smem);
      float* Tt = Tp + TC_BM * TS;
      {
        const int t = threadIdx.x;
        if (t < TC_BM) {
          const int ii = m0 + t;
          bulk_one(Tp + t * TS, S.GS + ((long)z * b + ii) * b + n0, ii < b ? (uint32_t)(BN * 4) : 0u);
        } else if (t < TC_BM + BN) {
          const int cc = t - TC_BM;
          bulk_one(Tt + cc * TP, S.GS + ((long)z * b + n0 + cc) * b + m0, (uint32_t)(min(TC_BM, b - m0) * 4));
        } else {
          bulk_one(nullptr, nullptr, 0u);
        }
      }
      bool got = mbar_wait(ew_bar, ew_phase, KID_CNP_FUSED, 5);
      ew_phase ^= 1u;
      got = __syncthreads_and(got);
      if (got) {
        for (int r = warp; r < TC_BM; r += CNP_THREADS / 32) {
          const int ii = m0 + r;
          if (ii >= b) break;
          for (int cc = lane; cc < BN; cc += 32) {
            const int jj = n0 + cc;
            if (ii < jj) S.grad[(long)z * P + packed_pos(ii, jj, b)] = Tp[r * TS + cc] - Tt[cc * TP + r];
          }
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
