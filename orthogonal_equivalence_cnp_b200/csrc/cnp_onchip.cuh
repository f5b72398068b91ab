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
// (the pair's off-diagonal quadrant crosses over once) and writes the packed rows coalesced.
//
// Synchronisation.  One thread of the (even) CTA issues every product once all epilogue warps
// of the pair have arrived on its `ready` barrier (release at cluster scope after their shared
// memory writes, TMEM stores and proxy fences); the product's completion is committed to the
// `mma` barrier of both CTAs.  Every wait is bounded (a timeout records the device error word,
// and the kernel skips the rest of its work but still runs every cluster barrier and frees TMEM).
#pragma once

#include "common.cuh"
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
  static constexpr int PITCH = B + 1;              // transposed-tile pitch of PACK (floats)
  static constexpr size_t SMEM = 3 * (size_t)REG + 1024 + 256;
  static_assert((size_t)B * (B - 1) / 2 * 4 <= 2 * (size_t)REG, "theta staging fits V1 + V2");
  static_assert((size_t)ROWS * PITCH * 4 <= 3 * (size_t)REG, "PACK tile fits the operand buffers");
};

struct CnpChipSide {
  CUtensorMap tmQ;      // forward: store map of Q [nb*b, b] bf16, 128-byte swizzle, box 64 x rows
  const float* theta;   // [nb, b(b-1)/2]
  const float* part;    // adjoint: split-K partials of G = dL/dQ, [splits][nb*b][b] fp32
  float* grad;          // adjoint: packed gradients [nb, b(b-1)/2]
  int nb;
  int splits;
};
struct CnpChipArgs {
  CnpChipSide seg[2];
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
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = smem_u32(smem);
  const uint32_t SC = s0, V1 = s0 + C::REG, V2 = s0 + 2 * C::REG;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 3 * C::REG);
  const uint32_t bar_mma = smem_u32(bars), bar_ready = smem_u32(bars + 1), bar_theta = smem_u32(bars + 2);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bars + 4);

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

  if (threadIdx.x == 0) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_ready, 8 * C::NCTA);
    mbar_init(bar_theta, 1);
    fence_mbar_init();
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
  griddep_wait();  // theta and the gradient partials come from earlier kernels

  bool ok = true;
  uint32_t mma_phase = 0, ready_phase = 0;

  // All epilogue warps of the pair report that their writes for the next product are done.
  auto arrive_ready = [&]() {
    fence_proxy_async_all();
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if constexpr (C::PAIR) mbar_arrive_cluster(ready_dst); else mbar_arrive(bar_ready);
    }
  };
  // D = A . B^T (+ D) over K = b, A K-major (A form), B K-major (A form of its N rows) or
  // MN-major (B form); a_neg negates A.  Issued by one thread once the pair is ready.
  auto issue = [&](uint32_t a, uint32_t b_op, bool b_mn, bool a_neg, bool accumulate, int site) {
    if (leader && warp == 0) {
      if (lane == 0) {
        if (ok) ok = C::PAIR ? mbar_wait_cluster(bar_ready, ready_phase, KID_CNP_CHIP, site)
                             : mbar_wait(bar_ready, ready_phase, KID_CNP_CHIP, site);
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
  auto wait_mma = [&](int site) {
    if (ok) ok = mbar_wait(bar_mma, mma_phase, KID_CNP_CHIP, site);
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
  auto tst = [&](uint32_t col, const float (&v)[32]) {
    tmem_st_32x32b_x32(col, reinterpret_cast<const uint32_t(&)[32]>(v));
  };
  // Row i, columns j0..j0+31 of the B form: element (k = i, n = j) in the CTA owning column j.
  auto put_bform = [&](uint32_t buf, int j0, const float (&v)[32]) {
    const int ct = C::PAIR ? j0 / 128 : 0;
    const int nl = j0 - 128 * ct;
    uint32_t row = buf + (uint32_t)(nl / 64) * C::BFORM_ATOM + (uint32_t)i * 128u;
    if (C::PAIR && ct != c) row = mapa_shared(row, (uint32_t)ct);
    const int ch0 = (nl % 64) / 8;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 w = make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                 pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
      st_cluster_v4(row + (uint32_t)(((ch0 + u) ^ (i & 7)) * 16), w);
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
      bulk_wait<0>();
    }
  };

  // ---------------------------------------------------------------- theta -> S (Sc, REG2)
  const bool need_s = !ADJ || k >= 1;
  if (need_s) {
    if (warp == 0) {
      const uint32_t bytes = (uint32_t)(P * 4);  // 16-byte multiple for b % 8 == 0
      if (lane == 0) mbar_arrive_expect_tx(bar_theta, bytes);
      __syncwarp();
      const uint32_t chunk = ((bytes / 8) + 15) & ~15u;
      const uint32_t off = (uint32_t)lane * chunk;
      if (lane < 8 && off < bytes)
        bulk_load_1d(V1 + off, reinterpret_cast<const char*>(SD.theta + z * P) + off, min(chunk, bytes - off), bar_theta);
    }
    if (ok) ok = mbar_wait(bar_theta, 0, KID_CNP_CHIP, 1);
    const float* th = reinterpret_cast<const float*>(smem + C::REG);
    const int roi = ro(i);
#pragma unroll 1
    for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
      float v[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int j = j0 + u;
        // one unconditional shared load per element (element 0 where nothing is read)
        const int idx = (!valid || j == i) ? 0 : (j > i ? roi + j : ro(j) + i);
        const float x = th[idx];
        v[u] = (!valid || j == i) ? 0.f : (j > i ? x : -x);
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
    // Every CTA of the cluster has read its theta staging before V1 / V2 are written (the peer
    // writes into this CTA's V2).
    if constexpr (C::PAIR) cluster_sync_all(); else __syncthreads();
    const long sstride = (long)SD.nb * B * B;
#pragma unroll 1
    for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
      float g[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) g[u] = 0.f;
      if (valid) {
        for (int sp = 0; sp < SD.splits; ++sp) {
          const float4* src = reinterpret_cast<const float4*>(SD.part + sp * sstride + (z * B + i) * B + j0);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float4 f = __ldg(src + u);
            g[4 * u] += f.x; g[4 * u + 1] += f.y; g[4 * u + 2] += f.z; g[4 * u + 3] += f.w;
          }
        }
      }
      tst(REG2 + j0, g);
      if (k >= 1) {
        chip_put_aform(V1, r, j0, g);  // R_k = G
        if (valid) put_bform(V2, j0, g);  // L_k = G
      }
    }
    uint32_t fcol = REG2;  // the TMEM columns holding G_S for PACK
    if (k >= 1) {
      fcol = ACC;
#pragma unroll 1
      for (int a = k - 1; a >= 0; --a) {
        arrive_ready();
        issue(V1, SC, false, false, false, 6);  // ACC = R_{a+1} . S^T = R_{a+1} T
        wait_mma(7);
#pragma unroll 1
        for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
          float d[32], g[32];
          tld(ACC + j0, d);
          tld(REG2 + j0, g);
#pragma unroll
          for (int u = 0; u < 32; ++u) d[u] += 2.f * g[u];  // R_a
          tst(ACC + j0, d);
          if (a > 0) chip_put_aform(V1, r, j0, d);
        }
        arrive_ready();
        issue(SC, V2, true, true, true, 8);  // ACC += (-S) . L_{a+1} = T L_{a+1}
        wait_mma(9);
        if (a > 0) {
#pragma unroll 1
          for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
            float l[32];
            tld(ACC + j0, l);
            if (valid) put_bform(V2, j0, l);
          }
        }
      }
    } else {
      tmem_wait_st();
    }
    griddep_launch();
    // ---------------------------------------------------------------------------- PACK
    // TT[i - rbase][j] = G_S[j][i] for this CTA's rows i and every j (pitch b + 1 floats).  A pair's
    // CTA 1 also sends CTA 0 the quadrant G_S[O_1][O_0]; CTA 0 keeps G_S[O_0][O_1] to itself
    // (CTA 1's packed rows only reach columns of O_1).
    {
      const int ct = C::PAIR ? c0 / 128 : 0;
      const bool send = !(C::PAIR && c == 0 && ct == 1) && valid;
      const uint32_t tt = (C::PAIR && ct != c) ? mapa_shared(s0, (uint32_t)ct) : s0;
#pragma unroll 1
      for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
        float f[32];
        tld(fcol + j0, f);
        if (send) {
#pragma unroll
          for (int u = 0; u < 32; ++u)
            st_cluster_f32(tt + (uint32_t)(((j0 + u - 128 * ct) * C::PITCH + i) * 4), f[u]);
        }
      }
    }
    if constexpr (C::PAIR) cluster_sync_all(); else __syncthreads();
    float* TT = reinterpret_cast<float*>(smem);
#pragma unroll 1
    for (int j0 = c0; j0 < c0 + C::HALF; j0 += 32) {
      float f[32];
      tld(fcol + j0, f);
      if (valid) {
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int j = j0 + u;
          if (j > i) TT[r * C::PITCH + j] = f[u] - TT[r * C::PITCH + j];
        }
      }
    }
    __syncthreads();
    if (ok) {
      float* out = SD.grad + z * P;
#pragma unroll 1
      for (int rr = warp; rr < C::ROWS; rr += 8) {
        const int ii = rbase + rr;
        const int base = ro(ii);
        for (int j = ii + 1 + lane; j < B; j += 32) out[base + j] = TT[rr * C::PITCH + j];
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
