// On-chip Cayley–Neumann kernels (bf16 tensor-core path, b = 64, 128, 256): the CNP forward and
// its adjoint for every block of one or two block sets in one launch, with every operand held in
// shared memory and every accumulator in TMEM (replication review of POET-X, "Summary": a fused
// kernel for the Cayley–Neumann series that reuses the lower powers; "Reproducibility & code":
// the forward and grad-Q kernels, k = 3).
//
// Ownership.  A 256-block belongs to a cluster of two CTAs that run tcgen05 as a pair
// (cta_group::2, M = 256): CTA c owns block rows O_c = [128c, 128c + 128).  A 64- or 128-block
// belongs to one CTA (M = 128; rows at or beyond b are padding).  Each CTA keeps in shared
// memory, as bf16 in the 128-byte-swizzled K-major layout ("A form": row r of its rows at
// r * 128 bytes of every 64-column atom):
//   Sc   the rows O_c of S.  For a pair this is also the K-major B half of any product X . S^T
//        (B columns n in O_c are rows n of S), and the A operand of any product S . X;
//   V1   the rows O_c of a varying left factor (A form) or of a symmetric right factor;
//   V2   a varying left factor (A form), or a varying right factor in MN-major form ("B form":
//        all b rows k of the matrix, the columns n of this CTA's N half).
// Products are therefore either X . F with F = S or a symmetric matrix (both operands are this
// CTA's own rows: no data leaves the CTA) or S . X (the B form of X needs the rows of both CTAs:
// each CTA writes the quadrant the peer needs straight into the peer's shared memory).
//
// Forward (Q = (I + S) sum_{j<=k} S^j = I + 2(S + ... + S^k) + S^(k+1)).  With P2 = S^2 (one
// product), the polynomial is evaluated by Horner's rule in P2 with coefficients linear in S:
//   U = 2S + 2P2;   Y' = S (k even) or 2S + P2 (k odd);   D = Y' . P2;
//   repeat floor(k/2) - 1 times: Y' = U + D, D = Y' . P2;   Q = I + U + D
// (k = 1: Q = I + 2S + P2; k = 0: Q = I + S).  That is 1 + floor(k/2) products of b x b x b
// instead of k; the identity and the exact first-order term stay in fp32.
//
// Adjoint.  For Q = sum_j c_j S^j (c_0 = c_{k+1} = 1, c_1..c_k = 2) and G = dL/dQ the gradient
// with respect to a free S is  G_S = sum_{a+c <= k} w_{a+c} T^a G T^c  with T = S^T = -S and
// w_m = c_{m+1}; the packed gradient is g[p(i,j)] = G_S[i][j] - G_S[j][i] (i < j).  G_S is
// evaluated by two interleaved Horner chains, k levels of two products each:
//   R_k = G, R_a = 2G + R_{a+1} T           (right factors: operands are own rows)
//   L_k = G, L_a = R_a + T L_{a+1},  G_S = L_0   (left factor T: L in B form, quadrant exchange)
// L_a accumulates onto R_a in the same TMEM columns.  PACK transposes G_S through shared memory
// (half of the pair's off-diagonal quadrant crosses over each way, so that both CTAs write the
// same number of packed entries) and writes the packed rows coalesced.
//
// Synchronisation.  One thread of the (even) CTA issues every product once all epilogue warps
// of the pair have arrived on its `ready` barrier (each after its shared memory writes, TMEM
// stores and proxy fences; the odd CTA's arrivals are remote); the product's completion is committed to the
// `mma` barrier of both CTAs.  Every wait is bounded (a timeout records the device error word,
// and the kernel skips the rest of its work but still runs every cluster barrier and frees TMEM).
#pragma once

#include "common.cuh"
#include "elementwise.cuh"
#include "gemm.cuh"
#include "sm100.cuh"

namespace poetx {

enum : int { KID_CNP_CHIP = 6 };

template <int B>
struct ChipCfg {
  static constexpr bool PAIR = B == 256;
  static constexpr int NCTA = PAIR ? 2 : 1;
  static constexpr int ROWS = PAIR ? 128 : B;      // block rows owned by one CTA
  static constexpr int M = PAIR ? 256 : 128;       // MMA rows (padding rows of a 64-block are zero)
  static constexpr int HALF = B / 2;               // columns per thread (two warps per TMEM lane quarter)
  static constexpr uint32_t ATOM = 128 * 128;      // one 64-column atom of an A-form buffer (128 rows)
  static constexpr uint32_t REG = (B / 64) * ATOM; // one operand buffer
  static constexpr uint32_t BFORM_ATOM = B * 128;  // one 64-column atom of a B-form buffer (b rows)
  static constexpr int TCOLS = 2 * B;              // TMEM: ACC [0, b), REG2 [b, 2b)
  static constexpr uint32_t GBOX = ROWS * 128;     // G staging: one 32-column fp32 box of this CTA's rows
  static constexpr int QN = PAIR ? 128 : B;        // PACK quadrant: QN x QN fp32, rows at QPITCH floats
  static constexpr int QPITCH = QN + 4;
  // Pair only: XS, the staging of the quadrant sent to the peer's B form (two 16 KiB atoms).
  static constexpr uint32_t XS_OFF = 3 * REG;
  static constexpr uint32_t XS_BYTES = PAIR ? 2 * 128 * 128 : 0;
  static constexpr size_t BAR_OFF = 3 * (size_t)REG + XS_BYTES;
  static constexpr size_t SMEM = BAR_OFF + 256 + 1024;
  static_assert((size_t)(B / 32) * GBOX <= 2 * (size_t)REG, "G staging fits V1 + V2");
  static_assert((size_t)B * (B - 1) / 2 * 4 <= 2 * (size_t)REG, "theta staging fits V1 + V2");
  // PACK: Qd, and for a pair three 128 x 64 half quadrants (received, sent, kept) of 68-float rows.
  static_assert((size_t)QN * QPITCH * 4 + (PAIR ? 3 * 128 * 68 * 4 : 0) <= BAR_OFF, "PACK staging fits below the barriers");
};

struct CnpChipSide {
  CUtensorMap tmQ;      // forward: store map of Q [nb*b, b] bf16, 128-byte swizzle, box 64 x rows
  CUtensorMap tmG;      // adjoint: load map of the partials [splits*nb*b, b] fp32, 128-byte swizzle,
                        //          box 32 x rows
  const float* theta;   // [nb, b(b-1)/2]
  const float* part;    // adjoint: split-K partials of G = dL/dQ, [splits][nb*b][b] fp32
  float* grad;          // adjoint: packed gradients [nb, b(b-1)/2]
  int nb;
  int splits;
};
// Spare blocks of a launch: the blocks past the CNP ones permute the columns of a bf16 row-major
// array, as permute_cols_bulk_kernel does, on the SMs the CNP leaves free (the forward's input
// gather U = X[:, pi_R], the adjoint's scatter of dU into dX), with a deeper ring (one block per
// SM there, and the CNP's shared memory to fill).
constexpr int kSpareSlots = 4;
struct CnpGather {
  const uint16_t* in;
  long ld_in;
  uint16_t* out;
  long ld_out;
  long rows;
  const int32_t* colmap;
  int cols;
  int scatter;  // 0: out[r][j] = in[r][colmap[j]];  1: out[r][colmap[j]] = in[r][j]
  int nblk;     // number of spare blocks (0: none)
};
struct CnpChipArgs {
  CnpChipSide seg[2];
  CnpGather gather;
  int ncnp;  // blocks of the CNP proper; blocks from ncnp on run the gather
  int nseg;
  int k;
};

// One 32-column chunk of a row as bf16 in an A-form buffer: row r, columns j0..j0+31 (j0 % 32 == 0).
__device__ __forceinline__ void chip_put_aform(uint32_t buf, int r, int j0, const float (&v)[32]) {
  const uint32_t row = buf + (uint32_t)(j0 / 64) * (128u * 128u) + (uint32_t)r * 128u;
  const int ch0 = (j0 % 64) / 8;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint4 w = make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                               pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
    const uint32_t a = row + (uint32_t)(((ch0 + u) ^ (r & 7)) * 16);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w)
                 : "memory");
  }
}

template <int B, bool ADJ>
__global__ void __launch_bounds__(256, 1) cnp_chip_kernel(const __grid_constant__ CnpChipArgs args) {
  using C = ChipCfg<B>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned start, derived by pointer arithmetic so that every pointer below stays in
  // the shared address space (32-bit shared loads instead of generic ones).
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t s0 = smem_u32(smem);
  const uint32_t SC = s0, V1 = s0 + C::REG, V2 = s0 + 2 * C::REG;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  const uint32_t bar_mma = smem_u32(bars), bar_ready = smem_u32(bars + 1), bar_theta = smem_u32(bars + 2);
  const uint32_t bar_g = smem_u32(bars + 3);
  const uint32_t bar_xin = smem_u32(bars + 4);  // data sent by the peer has landed here
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 6);

  if ((int)blockIdx.x >= args.ncnp) {  // a spare block: permute rows (whole clusters, no TMEM)
    griddep_wait();
    const CnpGather& G = args.gather;
    permute_cols_bulk_body<4, kSpareSlots>(smem, (long)blockIdx.x - args.ncnp, G.nblk, G.in, G.ld_in, G.out,
                                           G.ld_out, G.rows, G.cols, G.colmap, nullptr, G.scatter);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int c = C::PAIR ? (int)cluster_ctarank() : 0;
  const bool leader = c == 0;
  const long zg = C::PAIR ? (long)(blockIdx.x >> 1) : (long)blockIdx.x;
  const int seg = (args.nseg > 1 && zg >= args.seg[0].nb) ? 1 : 0;
  const long z = seg ? zg - args.seg[0].nb : zg;
  const CnpChipSide& SD = args.seg[seg];
  const int k = args.k;
  const int r = quarter * 32 + lane;          // this thread's row among the CTA's 128
  const int rbase = C::PAIR ? 128 * c : 0;
  const int i = rbase + r;                    // its block row
  const bool valid = i < B;
  const long P = (long)B * (B - 1) / 2;
  const int c0 = half * C::HALF;              // first column of this thread's half
  auto ro = [](int x) { return x * B - (x * (x + 1)) / 2 - x - 1; };  // packed (x, y) at ro(x) + y

  const bool need_s = !ADJ || k >= 1;
  if (threadIdx.x == 0) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_ready, 8 * C::NCTA);
    mbar_init(bar_theta, 1);
    mbar_init(bar_g, 1);
    mbar_init(bar_xin, 1);
    fence_mbar_init();
    if (need_s) {
      // The block's packed theta (8 bulk copies into V1 + V2) is requested first, so that the
      // TMEM allocation and the cluster barrier below overlap the copy.
      // The forward's theta may come from the launch just before (an optimiser step).  The
      // adjoint's never does (the launches before it are the layer's own backward products), so
      // it is read, and S built, while that launch finishes; only G waits for it.
      if (!ADJ) griddep_wait();
      const uint32_t bytes = (uint32_t)(P * 4);  // 16-byte multiple for b % 8 == 0
      mbar_arrive_expect_tx(bar_theta, bytes);
      const uint32_t chunk = ((bytes / 8) + 15) & ~15u;
#pragma unroll 1
      for (uint32_t off = 0; off < bytes; off += chunk)
        bulk_load_1d(V1 + off, reinterpret_cast<const char*>(SD.theta + z * P) + off, min(chunk, bytes - off), bar_theta);
    }
  }
  if (warp == 0) {
    if constexpr (C::PAIR) {
      tmem_alloc_pair(smem_u32(holder), C::TCOLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(holder), C::TCOLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (C::PAIR) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *holder;  // lane 0, column 0: the accumulator address of every product
  const uint32_t tlane = tbase + ((uint32_t)(quarter * 32) << 16);
  const uint32_t ACC = tlane, REG2 = tlane + B;
  const uint32_t ready_dst = (C::PAIR && !leader) ? mapa_shared(bar_ready, 0) : bar_ready;
  if (!ADJ) griddep_wait();  // Q is written over what earlier kernels may still read

  bool ok = true;
  uint32_t mma_phase = 0, ready_phase = 0, xin_phase = 0;
  const uint32_t peer = (uint32_t)(c ^ 1);

  // All epilogue warps of the pair report that their writes for the next product are done.
  // After an exchange (xin), the odd CTA's warp 0 first waits for the peer's data to land in its
  // own B form, so that the leader's `ready` also stands for that data.
  auto arrive_ready = [&](bool xin = false) {
    fence_proxy_async_smem();  // every operand write is to this CTA's own shared memory
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if constexpr (C::PAIR) {
        if (xin && c == 1 && warp == 0 && ok) ok = mbar_wait_cluster(bar_xin, xin_phase & 1u, KID_CNP_CHIP, 11);
        mbar_arrive_cluster(ready_dst);
      } else {
        mbar_arrive(bar_ready);
      }
    }
    if (xin) ++xin_phase;
  };
  // D = A . B^T (+ D) over K = b, A K-major (A form), B K-major (A form of its N rows) or
  // MN-major (B form); a_neg negates A.  Issued by one thread once the pair is ready.
  // xin: the B operand is a B form just exchanged; the leader also waits for its own incoming half
  // (the odd CTA's was folded into its `ready` arrival).  Call after arrive_ready(true).
  auto issue = [&](uint32_t a, uint32_t b_op, bool b_mn, bool a_neg, bool accumulate, int site, bool xin = false) {
    if (leader && warp == 0) {
      if (lane == 0) {
        if (ok) ok = C::PAIR ? mbar_wait_cluster(bar_ready, ready_phase, KID_CNP_CHIP, site)
                             : mbar_wait(bar_ready, ready_phase, KID_CNP_CHIP, site);
        if (C::PAIR && xin && ok) ok = mbar_wait_cluster(bar_xin, (xin_phase - 1) & 1u, KID_CNP_CHIP, 12);
        if (ok) {
          tc_fence_after();
          const uint32_t idesc = idesc_bf16_f32(C::M, B, false, b_mn) | (a_neg ? (1u << 13) : 0u);
#pragma unroll 1
          for (int kk = 0; kk < B / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(a + (uint32_t)(kk / 4) * C::ATOM + (uint32_t)(kk % 4) * 32, 16, 1024);
            const uint64_t bd = b_mn ? smem_desc_sw128(b_op + (uint32_t)kk * 2048, C::BFORM_ATOM, 1024)
                                     : smem_desc_sw128(b_op + (uint32_t)(kk / 4) * C::ATOM + (uint32_t)(kk % 4) * 32, 16, 1024);
            if constexpr (C::PAIR) mma_bf16_pair(tbase, ad, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
            else mma_bf16(tbase, ad, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
          }
          if constexpr (C::PAIR) mma_commit_pair(bar_mma, 0x3); else mma_commit(bar_mma);
        }
      }
      __syncwarp();
    }
    ready_phase ^= 1u;
  };
  // Every wait ends in a full-warp vote, so that the warp is converged (and agrees on `ok`)
  // before the warp-collective TMEM accesses that follow.
  auto wait_mma = [&](int site) {
    if (ok) ok = mbar_wait(bar_mma, mma_phase, KID_CNP_CHIP, site);
    ok = __all_sync(0xffffffffu, ok);
    mma_phase ^= 1u;
    tc_fence_after();
  };
  // 32 columns j0.. of this thread's TMEM row.
  auto tld = [&](uint32_t col, float (&v)[32]) {
    uint32_t w[32];
    tmem_ld_32x32b_x32(col, w);
    tmem_wait_ld();
#pragma unroll
    for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(w[u]);
  };
  auto tld2 = [&](uint32_t col1, float (&v1)[32], uint32_t col2, float (&v2)[32]) {
    uint32_t w1[32], w2[32];
    tmem_ld_32x32b_x32(col1, w1);
    tmem_ld_32x32b_x32(col2, w2);
    tmem_wait_ld();
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      v1[u] = __uint_as_float(w1[u]);
      v2[u] = __uint_as_float(w2[u]);
    }
  };
  auto tst = [&](uint32_t col, const float (&v)[32]) {
    tmem_st_32x32b_x32(col, reinterpret_cast<const uint32_t(&)[32]>(v));
  };
  // Row i, columns j0..j0+31 of the B form: element (k = i, n = j) in the CTA owning column j.
  // The peer's columns go to XS, laid out as the peer's B-form rows of this CTA's rows, and
  // leave in one exchange (send_bform) once every warp has written them.
  auto put_bform = [&](uint32_t buf, int j0, const float (&v)[32]) {
    const int ct = C::PAIR ? j0 / 128 : 0;
    const int nl = j0 - 128 * ct;
    const uint32_t row = (C::PAIR && ct != c) ? s0 + C::XS_OFF + (uint32_t)(nl / 64) * (128u * 128u) + (uint32_t)r * 128u
                                              : buf + (uint32_t)(nl / 64) * C::BFORM_ATOM + (uint32_t)i * 128u;
    const int ch0 = (nl % 64) / 8;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 w = make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                 pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + (uint32_t)(((ch0 + u) ^ (i & 7)) * 16)),
                   "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w)
                   : "memory");
    }
  };
  // The exchange of a B form written by put_bform (pair only; every thread calls it): the peer
  // expects 32 KiB on its xin barrier; this CTA's XS (rows O_c of the peer's two column atoms)
  // goes out as two 16 KiB copies into the peer's buffer `buf`.  Only the four warps holding the
  // peer's column half wrote XS, so only they meet before the copy: the leader's warp 0, which
  // may still be blocked issuing the product that runs meanwhile, is not waited for.
  auto send_bform = [&](uint32_t buf) {
    if constexpr (C::PAIR) {
      if (half == (c ^ 1)) {
        fence_proxy_async_smem();  // XS was written by the generic proxy; the copy engine reads it
        named_bar_sync(1, 128);
        if (quarter == 0 && lane == 0) {
          mbar_arrive_expect_tx(bar_xin, 2u * 128u * 128u);  // this CTA's incoming half
          const uint32_t bar_peer = mapa_shared(bar_xin, peer);
#pragma unroll
          for (int t = 0; t < 2; ++t)
            bulk_copy_to_peer(mapa_shared(buf + (uint32_t)t * C::BFORM_ATOM + (uint32_t)(128 * c) * 128u, peer),
                              s0 + C::XS_OFF + (uint32_t)t * (128u * 128u), 128u * 128u, bar_peer);
        }
      }
    }
  };
  // Q rows of this CTA leave through TMA stores of the A-form staging in V2.
  auto store_q = [&]() {
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0 && ok) {
#pragma unroll 1
      for (int a = 0; a < B / 64; ++a) tma_store_2d(&SD.tmQ, V2 + (uint32_t)a * C::ATOM, 64 * a, (int)(z * B + rbase));
      bulk_commit();
      bulk_wait_read<0>();  // the staging may be released; the stores complete with the grid
    }
  };

  // ---------------------------------------------------------------- theta -> S (Sc, REG2)
  if (need_s) {
    if (ok) ok = mbar_wait(bar_theta, 0, KID_CNP_CHIP, 1);
    ok = __all_sync(0xffffffffu, ok);
    const float* th = reinterpret_cast<const float*>(smem + C::REG);
    const int roi = ro(i);
    const int iw = rbase + quarter * 32;  // first row of this warp: chunks are warp-uniform
#pragma unroll 1
    for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
      float v[32];
      if (!valid) {
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = 0.f;
      } else if (j0 >= iw + 32) {
        // above the diagonal for every lane: S[i][j] = theta[p(i, j)], contiguous in j
        const float* src = th + roi + j0;
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = src[u];
      } else if (j0 + 32 <= iw) {
        // below it: S[i][j] = -theta[p(j, i)]; p(j, i) = ro(j) + i with ro(j+1) = ro(j) + b - 2 - j
        const float* src = th + ro(j0) + i;
        const int step0 = B - 2 - j0;
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = -src[u * step0 - (u * (u - 1)) / 2];
      } else {
        // The warp's diagonal block: both candidates are loaded at offsets that are the same for
        // every lane (the one not selected is a harmless shared-memory read: at worst one float
        // before the staging, for row 0), then selected.
        const float* up = th + roi + j0;
        const float* lo = th + ro(j0) + i;
        const int step0 = B - 2 - j0;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const float xu = up[u];
          const float xl = lo[u * step0 - (u * (u - 1)) / 2];
          const int j = j0 + u;
          v[u] = j > i ? xu : (j < i ? -xl : 0.f);
        }
      }
      chip_put_aform(SC, r, j0, v);
      if constexpr (!ADJ) tst(REG2 + j0, v);
    }
  }

  if constexpr (!ADJ) {
    // ------------------------------------------------------------------------- forward
    const int nst = k / 2;  // Horner steps in P2 after the product P2 = S^2
    if (k == 0) {
      __syncthreads();  // every warp has read the theta staging, which V2 overlaps
      tmem_wait_st();
#pragma unroll 1
      for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
        float s[32];
        tld(REG2 + j0, s);
#pragma unroll
        for (int u = 0; u < 32; ++u) s[u] += (i == j0 + u) ? 1.f : 0.f;
        if (valid) chip_put_aform(V2, r, j0, s);
      }
      griddep_launch();
      store_q();
    } else {
      arrive_ready();
      issue(SC, SC, false, false, false, 2);  // ACC = S . S^T = -P2
      wait_mma(3);
#pragma unroll 1
      for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
        float d[32], s[32], o[32];
        tld(ACC + j0, d);
        tld(REG2 + j0, s);
        if (k == 1) {
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = 2.f * s[u] - d[u] + ((i == j0 + u) ? 1.f : 0.f);
          if (valid) chip_put_aform(V2, r, j0, o);
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = -d[u];
          chip_put_aform(V1, r, j0, o);  // P2 (symmetric: its rows are the K-major B operand)
          if (k & 1) {
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = 2.f * s[u] - d[u];
            chip_put_aform(V2, r, j0, o);  // Y' = 2S + P2
          }
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = 2.f * s[u] - 2.f * d[u];
          tst(REG2 + j0, o);  // U = 2S + 2P2
        }
      }
      if (k == 1) {
        griddep_launch();
        store_q();
      } else {
#pragma unroll 1
        for (int t = 0; t < nst; ++t) {
          const bool last = t == nst - 1;
          arrive_ready();
          issue((t == 0 && !(k & 1)) ? SC : V2, V1, false, false, false, 4);  // D = Y' . P2
          wait_mma(5);
          if (last) griddep_launch();
#pragma unroll 1
          for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
            float d[32], u2[32];
            tld(ACC + j0, d);
            tld(REG2 + j0, u2);
#pragma unroll
            for (int u = 0; u < 32; ++u) d[u] += u2[u] + ((last && i == j0 + u) ? 1.f : 0.f);
            if (!last || valid) chip_put_aform(V2, r, j0, d);  // next Y' = U + D, or Q = I + U + D
          }
          if (last) store_q();
        }
      }
    }
  } else {
    // ------------------------------------------------------------------------- adjoint
    // G = sum of the split-K partials -> REG2 (fp32).  Each partial's rows of this CTA arrive as
    // b/32 TMA boxes (32 columns x rows, 128-byte swizzle: the 16-byte chunk q of row r sits at
    // position q ^ (r % 8)), one round per partial, so that every thread then reads its own row
    // with conflict-free 16-byte loads.  The staging overlaps V1 / V2 (and the theta staging):
    // every CTA of the cluster has finished its theta reads before the first round starts.
    if constexpr (C::PAIR) cluster_sync_all(); else __syncthreads();
    griddep_wait();  // the partials come from the launch just before
#pragma unroll 1
    for (int sp = 0; sp < SD.splits; ++sp) {
      if (sp > 0) __syncthreads();  // every thread has read the previous round
      if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar_g, (uint32_t)(C::ROWS * B * 4));
#pragma unroll 1
        for (int a = 0; a < B / 32; ++a)
          tma_load_2d(V1 + (uint32_t)a * C::GBOX, &SD.tmG, bar_g, 32 * a, (int)(((long)sp * SD.nb + z) * B + rbase));
      }
      if (ok) ok = mbar_wait(bar_g, (uint32_t)(sp & 1), KID_CNP_CHIP, 10);
      ok = __all_sync(0xffffffffu, ok);
#pragma unroll 1
      for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
        float g[32];
        if (sp > 0) tld(REG2 + j0, g);
        const uint8_t* row = smem + C::REG + (j0 / 32) * C::GBOX + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 f = valid ? *reinterpret_cast<const float4*>(row + ((u ^ (r & 7)) * 16))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
          if (sp > 0) {
            g[4 * u] += f.x; g[4 * u + 1] += f.y; g[4 * u + 2] += f.z; g[4 * u + 3] += f.w;
          } else {
            g[4 * u] = f.x; g[4 * u + 1] = f.y; g[4 * u + 2] = f.z; g[4 * u + 3] = f.w;
          }
        }
        tst(REG2 + j0, g);
      }
      tmem_wait_st();
    }
    // R_k = G (A form in V1) and L_k = G (B form in V2, the peer's quadrant in the peer): every
    // CTA of the cluster has finished reading its G staging.
    if constexpr (C::PAIR) cluster_sync_all(); else __syncthreads();
    uint32_t fcol = REG2;  // the TMEM columns holding G_S for PACK
    if (k >= 1) {
      // Each product is issued as soon as its operands are in place; the rest of an epilogue (the
      // bf16 copies that only a later product reads, and the exchange) runs beside it:
      //   R_a = ACC + 2G goes back into ACC first (MMA_L accumulates onto it), its A form into V1
      //   while MMA_L runs; L_a is read out of ACC, then MMA_R of the next level may overwrite ACC
      //   while L_a's B form is written and exchanged.  The first product needs only R_k = G in
      //   A form, so L_k = G's B form is written and exchanged beside it.
      constexpr int NCH = C::HALF / 32;  // 32-column chunks per thread
      fcol = ACC;
      {
        float gv[NCH][32];
#pragma unroll
        for (int q = 0; q < NCH; ++q) {
          tld(REG2 + c0 + 32 * q, gv[q]);
          chip_put_aform(V1, r, c0 + 32 * q, gv[q]);
        }
        arrive_ready();
        issue(V1, SC, false, false, false, 6);  // ACC = R_k . S^T = R_k T
#pragma unroll
        for (int q = 0; q < NCH; ++q)
          if (valid) put_bform(V2, c0 + 32 * q, gv[q]);
        send_bform(V2);
      }
#pragma unroll 1
      for (int a = k - 1; a >= 0; --a) {
        wait_mma(7);
        float rv[NCH][32];
#pragma unroll
        for (int q = 0; q < NCH; ++q) {
          float g[32];
          tld2(ACC + c0 + 32 * q, rv[q], REG2 + c0 + 32 * q, g);
#pragma unroll
          for (int u = 0; u < 32; ++u) rv[q][u] += 2.f * g[u];  // R_a
          tst(ACC + c0 + 32 * q, rv[q]);
        }
        arrive_ready(true);  // ACC = R_a; MMA_L reads V2 = L_{a+1}, the B form exchanged after its epilogue
        issue(SC, V2, true, true, true, 8, true);  // ACC += (-S) . L_{a+1} = T L_{a+1}
        if (a > 0) {
#pragma unroll
          for (int q = 0; q < NCH; ++q) chip_put_aform(V1, r, c0 + 32 * q, rv[q]);  // R_a for the next level
        }
        wait_mma(9);
        if (a > 0) {
          float lv[NCH][32];
#pragma unroll
          for (int q = 0; q < NCH; ++q) tld(ACC + c0 + 32 * q, lv[q]);  // L_a
          arrive_ready();  // L_a is out of ACC and R_a is in V1
          issue(V1, SC, false, false, false, 6);  // ACC = R_a . S^T = R_a T (next level)
#pragma unroll
          for (int q = 0; q < NCH; ++q)
            if (valid) put_bform(V2, c0 + 32 * q, lv[q]);
          send_bform(V2);
        }
      }
    } else {
      tmem_wait_st();
    }
    griddep_launch();
    // ---------------------------------------------------------------------------- PACK
    // g[p(i,j)] = G_S[i][j] - G_S[j][i] for i < j, written along j (lanes take consecutive j) so
    // that every packed row p(i, .) leaves as coalesced stores.  Qd = G_S[O_c][O_c] (QN x QN, rows
    // of QPITCH floats) is staged by the threads holding it; the thread owning row j of a diagonal
    // quadrant reads G_S[j][i] from TMEM and G_S[i][j] from Qd.  For a pair, the cross quadrant
    // (i in O_0, j in O_1) is split in two halves of 64 columns j, one per CTA, so that both do the
    // same amount of work: CTA 1 takes j in [128, 192) (G_S[j][i] from its TMEM, G_S[i][j] sent by
    // CTA 0), CTA 0 takes j in [192, 256) (G_S[i][j] staged from its TMEM, G_S[j][i] sent by CTA 1
    // transposed).  Both halves cross in one bulk copy each way (XPITCH-float rows).
    {
      constexpr int XPITCH = 68;                            // 64 columns + 4 (16-byte rows)
      constexpr uint32_t XBYTES = 128u * XPITCH * 4u;       // one 128 x 64 half quadrant
      const uint32_t QD = s0;
      const uint32_t RX = s0 + (uint32_t)(C::QN * C::QPITCH * 4);  // received half quadrant
      const uint32_t SX = RX + XBYTES;                              // half quadrant sent to the peer
      const uint32_t XL = SX + XBYTES;                              // CTA 0: G_S[O_0][192..255] kept here
      const int own0 = C::PAIR ? 128 * c : 0;  // first column of this CTA's own quadrant
      const bool own_cols = !C::PAIR || half == c;
#pragma unroll 1
      for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
        float f[32];
        tld(fcol + j0, f);
        if (!valid) continue;
        uint32_t at = 0;
        if (own_cols) at = QD + (uint32_t)(r * C::QPITCH + (j0 - own0)) * 4u;
        else if (C::PAIR && c == 0) at = (j0 < 192 ? SX + (uint32_t)(r * XPITCH + (j0 - 128)) * 4u
                                                   : XL + (uint32_t)(r * XPITCH + (j0 - 192)) * 4u);
        if (own_cols || (C::PAIR && c == 0)) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(at + 16 * u), "r"(__float_as_uint(f[4 * u])),
                         "r"(__float_as_uint(f[4 * u + 1])), "r"(__float_as_uint(f[4 * u + 2])),
                         "r"(__float_as_uint(f[4 * u + 3]))
                         : "memory");
        } else if (C::PAIR && i >= 192) {
          // CTA 1, rows j in [192, 256): G_S[j][i] for i = j0.. into column j - 192 of the transposed
          // staging (lanes write consecutive floats).
          const uint32_t colp = SX + (uint32_t)(j0 * XPITCH + (i - 192)) * 4u;
#pragma unroll
          for (int u = 0; u < 32; ++u)
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(colp + (uint32_t)(u * XPITCH * 4)), "f"(f[u]) : "memory");
        }
      }
      if (C::PAIR && threadIdx.x == 0) mbar_arrive_expect_tx(bar_xin, XBYTES);
      fence_proxy_async_smem();
      __syncthreads();
      if (C::PAIR && threadIdx.x == 0) bulk_copy_to_peer(mapa_shared(RX, peer), SX, XBYTES, mapa_shared(bar_xin, peer));
      const int j = i;
      const int jwarp = rbase + quarter * 32;  // first row of this warp
      float* out = SD.grad + z * P;
      // Items of 32 rows i against this warp's 32 rows j: the diagonal quadrant's chunks below the
      // warp's rows, then (once the peer's half quadrant has landed) in CTA 1 for j < 192 the four
      // chunks of O_0.  The two warps of a lane quarter take them in turn.  The TMEM loads are
      // warp-collective: the chunk list is the same for every lane, and i < j only guards the stores.
      const int ndiag = jwarp < B ? (jwarp - own0) / 32 + 1 : 0;  // warps past row b - 1 (b = 64) have none
      const int ncross = (C::PAIR && c == 1 && jwarp < 192) ? 4 : 0;
      auto pack_item = [&](bool cross, int i0) {
        float f[32];
        tld(fcol + i0, f);  // G_S[j][i0 .. i0 + 31]
        // G_S[i0 + u][j] at qcol[u * pitch]; g[p(i0 + u, j)] at o_u, with p(i + 1, j) - p(i, j) = b - 2 - i.
        const float* qcol = cross ? reinterpret_cast<const float*>(smem + (RX - s0)) + i0 * XPITCH + (j - 128)
                                  : reinterpret_cast<const float*>(smem) + (i0 - own0) * C::QPITCH + (j - own0);
        const int pitch = cross ? XPITCH : C::QPITCH;
        const bool store = ok && valid;
        float* o = out + ro(i0) + j;
        int step = B - 2 - i0;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          if (store && i0 + u < j) *o = qcol[u * pitch] - f[u];
          o += step;
          --step;
        }
      };
#pragma unroll 1
      for (int item = half; item < ndiag; item += 2) pack_item(false, own0 + 32 * item);
      if (C::PAIR) {
        if (ok) ok = mbar_wait(bar_xin, xin_phase & 1u, KID_CNP_CHIP, 13);
        ok = __all_sync(0xffffffffu, ok);
      }
      ++xin_phase;
#pragma unroll 1
      for (int item = half; item < ncross; item += 2) pack_item(true, 32 * item);
      if (C::PAIR && c == 0) {
        // CTA 0's half of the cross quadrant, one 32 x 32 item per warp, entirely from shared
        // memory: G_S[i][j] (kept) minus G_S[j][i] (received transposed).
        const int i0 = 32 * (warp & 3);
        const int jx = 192 + 32 * (warp >> 2) + lane;
        const float* xl = reinterpret_cast<const float*>(smem + (XL - s0)) + i0 * XPITCH + (jx - 192);
        const float* yt = reinterpret_cast<const float*>(smem + (RX - s0)) + i0 * XPITCH + (jx - 192);
        float* o = out + ro(i0) + jx;
        int step = B - 2 - i0;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          if (ok) *o = xl[u * XPITCH] - yt[u * XPITCH];
          o += step;
          --step;
        }
      }
    }
  }

  tc_fence_before();
  if constexpr (C::PAIR) cluster_sync_all(); else __syncthreads();
  if (warp == 0) {
    if constexpr (C::PAIR) tmem_dealloc_pair(tbase, C::TCOLS); else tmem_dealloc(tbase, C::TCOLS);
  }
}

}  // namespace poetx
