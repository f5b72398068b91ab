// Memory-bound kernels of the POET-X layer: permutation of the feature dimension, packed skew
// unpack / packed-gradient pack, split-K reduction, permutation inverse and composition.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace poetx {

// Position of S[i][j] (i < j) in the packed upper triangle, row by row.
__host__ __device__ __forceinline__ long packed_pos(int i, int j, int b) {
  return (long)i * b - (long)i * (i + 1) / 2 + (j - i - 1);
}

// Index-based permutation of the feature (column) dimension of a row-major [rows, cols] array
// (replication review of POET-X, "Summary": permutations applied by index, never as a matmul;
// Table 1 of the paper measures such a kernel).  HBM sees one read and one write per element.
// ROWS rows (4, or 2 for very wide rows) are processed together and stored in shared memory
// interleaved: one word (ROWS x 16 bit) holds element c of all of them, so one random word
// access moves ROWS elements.  The word of column c sits at (c & 7) * (cols / 8) + (c >> 3),
// which lets the loading lanes write consecutive words (no bank conflicts).  Rows are read with
// coalesced 16-byte loads straight into registers and written back with 16-byte coalesced
// stores; the 16-bit source map (for a scatter: the inverse map, built in shared memory)
// is cached per block.
//   gather (scatter == 0): out[r][j] = in[rowmap ? rowmap[r] : r][colmap[j]]
//   scatter (scatter == 1): out[r][colmap[j]] = in[r][j]
// bf16 (16-bit) elements; requires cols <= 65536, cols % 8 == 0, 16-byte aligned rows.
template <int ROWS>
__host__ __device__ constexpr size_t permute_smem_bytes(int cols) {
  return ((size_t)cols * 2 + 15) / 16 * 16 + (size_t)cols * 2 * ROWS;
}

template <int ROWS>
__global__ void __launch_bounds__(256, ROWS == 4 ? 3 : 2)
    permute_cols_bf16_kernel(const uint16_t* __restrict__ in, long ld_in, uint16_t* __restrict__ out, long ld_out,
                             long rows, int cols, const int32_t* __restrict__ colmap,
                             const int32_t* __restrict__ rowmap, int scatter) {
  sm100::griddep_wait();
  using Word = typename std::conditional<ROWS == 4, uint64_t, uint32_t>::type;
  extern __shared__ __align__(16) uint8_t smem_perm[];
  uint16_t* src_of = reinterpret_cast<uint16_t*>(smem_perm);  // output column j reads source column src_of[j]
  Word* W = reinterpret_cast<Word*>(smem_perm + ((size_t)cols * 2 + 15) / 16 * 16);
  const int nvec = cols / 8;
  auto build_map = [&]() {
    // The map is read with 16-byte loads, four per thread in flight (cols % 8 == 0, 16-byte
    // aligned map), so building it costs about one L2 round trip.
    const int n4 = cols / 4;
    for (int base = 0; base < n4; base += 4 * (int)blockDim.x) {
      int4 t[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = base + u * (int)blockDim.x + (int)threadIdx.x;
        if (v < n4) t[u] = __ldg(reinterpret_cast<const int4*>(colmap) + v);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = base + u * (int)blockDim.x + (int)threadIdx.x;
        if (v >= n4) continue;
        const int m4[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * v + e;
          if (scatter) src_of[m4[e]] = (uint16_t)j; else src_of[j] = (uint16_t)m4[e];
        }
      }
    }
  };
  const long ngroups = (rows + ROWS - 1) / ROWS;
  // Source rows of group g (a short last group repeats its last row; only nr rows are stored).
  auto group_rows = [&](long g, long (&src_row)[ROWS]) {
    const long r0 = g * ROWS;
    const int nr = (int)min((long)ROWS, rows - r0);
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      const long rr = r0 + min(r, nr - 1);
      src_row[r] = (!scatter && rowmap) ? (long)__ldg(rowmap + rr) : rr;
    }
  };
  // 8 columns of each row per thread, column vectors c0 and c0 + blockDim.x.
  auto load = [&](long g, int c0, uint4 (&v)[2][ROWS]) {
    long src_row[ROWS];
    group_rows(g, src_row);
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const int c = c0 + u * (int)blockDim.x;
        if (c < nvec) v[u][r] = __ldg(reinterpret_cast<const uint4*>(in + src_row[r] * ld_in) + c);
      }
  };
  auto put = [&](int c0, const uint4 (&v)[2][ROWS]) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = c0 + u * (int)blockDim.x;
      if (c >= nvec) continue;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        Word w = 0;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) w |= (Word)reinterpret_cast<const uint16_t*>(&v[u][r])[q] << (16 * r);
        W[q * nvec + c] = w;
      }
    }
  };
  // Column vector c of the output rows, each element read through the source map.
  auto store = [&](long g) {
    const long r0 = g * ROWS;
    const int nr = (int)min((long)ROWS, rows - r0);
    for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
      const uint4 ix4 = reinterpret_cast<const uint4*>(src_of)[c];
      const uint16_t* ix = reinterpret_cast<const uint16_t*>(&ix4);
      Word w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) w[q] = W[(ix[q] & 7) * nvec + (ix[q] >> 3)];
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        if (r >= nr) break;
        uint16_t e[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) e[q] = (uint16_t)(w[q] >> (16 * r));
        reinterpret_cast<uint4*>(out + (r0 + r) * ld_out)[c] = *reinterpret_cast<const uint4*>(e);
      }
    }
  };

  if (nvec <= 2 * (int)blockDim.x) {
    // A whole group fits in two vectors per thread: software pipeline across groups.  The first
    // group's loads are in flight while the map is built, and each next group's loads while the
    // current group is gathered and stored, so HBM sees reads and writes at the same time.
    uint4 v[2][ROWS];
    long g = blockIdx.x;
    if (g < ngroups) load(g, threadIdx.x, v);
    build_map();
    for (; g < ngroups; g += gridDim.x) {
      put(threadIdx.x, v);
      __syncthreads();  // W (and, the first time, the map) complete
      if (g + gridDim.x < ngroups) load(g + gridDim.x, threadIdx.x, v);
      store(g);
      __syncthreads();  // W free again
    }
    return;
  }
  build_map();
  __syncthreads();
  for (long g = blockIdx.x; g < ngroups; g += gridDim.x) {
    for (int c0 = threadIdx.x; c0 < nvec; c0 += blockDim.x * 2) {
      uint4 v[2][ROWS];
      load(g, c0, v);
      put(c0, v);
    }
    __syncthreads();
    store(g);
    __syncthreads();
  }
}

// Bulk-copy variant (bf16, 16-byte aligned rows): one thread streams each group's ROWS source
// rows into a two-slot shared-memory ring with 1-D TMA bulk copies (cp.async.bulk, completion
// on an mbarrier), so the loads of a block's next two groups are in flight without holding any
// registers; the threads then interleave the slot into the word array W (16-byte, conflict-free
// shared reads) and gather/store exactly as above.  With two blocks per SM and about two groups
// per block, the whole input is requested at once.  Waits are bounded (device error word, kernel
// id KID_PERMUTE); a block that gives up still reaches every barrier and skips its stores.
enum : int { KID_PERMUTE = 3 };

template <int ROWS, int SLOTS = 2>
__host__ __device__ constexpr size_t permute_bulk_smem_bytes(int cols) {
  return SLOTS * (size_t)ROWS * cols * 2    // ring: SLOTS slots of ROWS rows
         + (size_t)cols * 2 * ROWS          // W: one word of ROWS elements per column
         + ((size_t)cols * 2 + 15) / 16 * 16  // source map
         + 8 * SLOTS + 48;                   // SLOTS mbarriers (+ padding)
}

// The body of the kernel below as a device function: block `bid` of `nblk` blocks (256 threads)
// permutes its share of the row groups, staging in `smem_bulk` (permute_bulk_smem_bytes<ROWS>(cols)
// bytes, 128-byte aligned).  It also serves the spare blocks of a CNP launch (cnp_onchip.cuh).
template <int ROWS, int SLOTS = 2>
__device__ __forceinline__ void permute_cols_bulk_body(uint8_t* smem_bulk, long bid, long nblk,
                                                       const uint16_t* __restrict__ in, long ld_in,
                                                       uint16_t* __restrict__ out, long ld_out, long rows, int cols,
                                                       const int32_t* __restrict__ colmap,
                                                       const int32_t* __restrict__ rowmap, int scatter) {
  using Word = typename std::conditional<ROWS == 4, uint64_t, uint32_t>::type;
  const size_t slot_bytes = (size_t)ROWS * cols * 2;
  uint8_t* ring = smem_bulk;
  Word* W = reinterpret_cast<Word*>(smem_bulk + SLOTS * slot_bytes);
  uint16_t* src_of = reinterpret_cast<uint16_t*>(smem_bulk + SLOTS * slot_bytes + (size_t)cols * 2 * ROWS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_bulk + SLOTS * slot_bytes + (size_t)cols * 2 * ROWS +
                                               ((size_t)cols * 2 + 15) / 16 * 16);
  const int nvec = cols / 8;
  const long ngroups = (rows + ROWS - 1) / ROWS;
  const uint32_t row_bytes = (uint32_t)cols * 2;

  // Thread 0: request the ROWS source rows of group g into ring slot `slot`.
  auto request = [&](long g, int slot) {
    const long r0 = g * ROWS;
    const int nr = (int)min((long)ROWS, rows - r0);
    const uint32_t bar = sm100::smem_u32(bars + slot);
    sm100::mbar_arrive_expect_tx(bar, (uint32_t)nr * row_bytes);
    for (int r = 0; r < nr; ++r) {
      const long sr = (!scatter && rowmap) ? (long)__ldg(rowmap + r0 + r) : r0 + r;
      sm100::bulk_load_1d(sm100::smem_u32(ring + (size_t)slot * slot_bytes + (size_t)r * row_bytes),
                          in + sr * ld_in, row_bytes, bar);
    }
  };

  if (threadIdx.x == 0) {
#pragma unroll
    for (int q = 0; q < SLOTS; ++q) sm100::mbar_init(sm100::smem_u32(bars + q), 1);
    sm100::fence_mbar_init();
#pragma unroll
    for (int q = 0; q < SLOTS; ++q)
      if (bid + q * nblk < ngroups) request(bid + q * nblk, q);
  }
  // Source map (overlaps the first copies).
  {
    const int n4 = cols / 4;
    for (int base = 0; base < n4; base += 4 * (int)blockDim.x) {
      int4 t[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = base + u * (int)blockDim.x + (int)threadIdx.x;
        if (v < n4) t[u] = __ldg(reinterpret_cast<const int4*>(colmap) + v);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = base + u * (int)blockDim.x + (int)threadIdx.x;
        if (v >= n4) continue;
        const int m4[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * v + e;
          if (scatter) src_of[m4[e]] = (uint16_t)j; else src_of[j] = (uint16_t)m4[e];
        }
      }
    }
  }
  __syncthreads();  // barriers initialised, map complete
  sm100::griddep_launch();

  bool ok = true;
  int i = 0;
#pragma unroll 1
  for (long g = bid; g < ngroups; g += nblk, ++i) {
    const int slot = i % SLOTS;
    const long r0 = g * ROWS;
    const int nr = (int)min((long)ROWS, rows - r0);
    const bool got = sm100::mbar_wait(sm100::smem_u32(bars + slot), (uint32_t)(i / SLOTS) & 1u, KID_PERMUTE, 1);
    ok = __syncthreads_and(got);
    if (!ok) break;  // block-uniform
    // Interleave the slot into W (rows past nr repeat the last row).
    {
      const uint8_t* sl = ring + (size_t)slot * slot_bytes;
      for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
        uint4 v[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r)
          v[r] = reinterpret_cast<const uint4*>(sl + (size_t)min(r, nr - 1) * row_bytes)[c];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          Word w = 0;
#pragma unroll
          for (int r = 0; r < ROWS; ++r) w |= (Word)reinterpret_cast<const uint16_t*>(&v[r])[q] << (16 * r);
          W[q * nvec + c] = w;
        }
      }
    }
    __syncthreads();  // W complete; the slot has been read by every thread
    if (threadIdx.x == 0 && g + SLOTS * nblk < ngroups) {
      sm100::fence_proxy_async_smem();  // the copy engine overwrites what the threads just read
      request(g + SLOTS * nblk, slot);
    }
    {
      for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
        const uint4 ix4 = reinterpret_cast<const uint4*>(src_of)[c];
        const uint16_t* ix = reinterpret_cast<const uint16_t*>(&ix4);
        Word w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) w[q] = W[(ix[q] & 7) * nvec + (ix[q] >> 3)];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
          if (r >= nr) break;
          uint16_t e[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) e[q] = (uint16_t)(w[q] >> (16 * r));
          reinterpret_cast<uint4*>(out + (r0 + r) * ld_out)[c] = *reinterpret_cast<const uint4*>(e);
        }
      }
    }
    __syncthreads();  // W free again
  }
  // A block that gave up (at its group i) waits, bounded, for the copies it still has in flight
  // (groups i .. i + SLOTS - 1) before its shared memory is released.
  if (!ok && threadIdx.x == 0) {
    long g = bid + (long)i * nblk;
    for (int k = i; k < i + SLOTS && g < ngroups; ++k, g += nblk)
      sm100::mbar_wait(sm100::smem_u32(bars + (k % SLOTS)), (uint32_t)(k / SLOTS) & 1u, KID_PERMUTE, 2);
  }
  __syncthreads();
}

template <int ROWS>
__global__ void __launch_bounds__(256, 2)
    permute_cols_bulk_kernel(const uint16_t* __restrict__ in, long ld_in, uint16_t* __restrict__ out, long ld_out,
                             long rows, int cols, const int32_t* __restrict__ colmap,
                             const int32_t* __restrict__ rowmap, int scatter) {
  sm100::griddep_wait();
  extern __shared__ __align__(128) uint8_t smem_bulk[];
  permute_cols_bulk_body<ROWS>(smem_bulk, blockIdx.x, gridDim.x, in, ld_in, out, ld_out, rows, cols, colmap, rowmap,
                               scatter);
}

// AdamW on packed parameters (decoupled weight decay), fp32: per parameter 16 bytes read
// (theta, g, m, v) and 12 written (theta, m, v), so HBM bound.  float4 grid-stride over the
// first n - n % 4 parameters, the tail by the first threads.
struct AdamwArgs {
  float eta;          // gamma * lr
  float beta1, beta2;
  float inv_bc1;      // 1 / (1 - beta1^t)
  float inv_sqrt_bc2; // 1 / sqrt(1 - beta2^t)
  float eps, decay;
};

__device__ __forceinline__ void adamw_one(float& th, float g, float& m, float& v, const AdamwArgs& a) {
  m = a.beta1 * m + (1.f - a.beta1) * g;
  v = a.beta2 * v + (1.f - a.beta2) * g * g;
  const float denom = sqrtf(v) * a.inv_sqrt_bc2 + a.eps;
  th = th - a.eta * (a.decay * th + (m * a.inv_bc1) / denom);
}

__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ theta, const float* __restrict__ grad,
                                                    float* __restrict__ m, float* __restrict__ v, long n,
                                                    const AdamwArgs a) {
  sm100::griddep_wait();
  const long n4 = n / 4;
  const long stride = (long)gridDim.x * blockDim.x;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 t4 = reinterpret_cast<const float4*>(theta)[i];
    const float4 g4 = __ldg(reinterpret_cast<const float4*>(grad) + i);
    float4 m4 = reinterpret_cast<const float4*>(m)[i];
    float4 v4 = reinterpret_cast<const float4*>(v)[i];
    adamw_one(t4.x, g4.x, m4.x, v4.x, a);
    adamw_one(t4.y, g4.y, m4.y, v4.y, a);
    adamw_one(t4.z, g4.z, m4.z, v4.z, a);
    adamw_one(t4.w, g4.w, m4.w, v4.w, a);
    reinterpret_cast<float4*>(theta)[i] = t4;
    reinterpret_cast<float4*>(m)[i] = m4;
    reinterpret_cast<float4*>(v)[i] = v4;
  }
  const long tail = 4 * n4 + (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tail < n) adamw_one(theta[tail], grad[tail], m[tail], v[tail], a);
}

// fp32 variant for the fp32 path (small layers): one row at a time, staged in shared memory.
__global__ void __launch_bounds__(256)
    permute_cols_f32_kernel(const float* __restrict__ in, long ld_in, float* __restrict__ out, long ld_out, long rows,
                            int cols, const int32_t* __restrict__ colmap, const int32_t* __restrict__ rowmap,
                            int scatter) {
  sm100::griddep_wait();
  extern __shared__ __align__(16) uint8_t smem_perm[];
  float* row = reinterpret_cast<float*>(smem_perm);
  for (long r = blockIdx.x; r < rows; r += gridDim.x) {
    const long rin = (!scatter && rowmap) ? (long)__ldg(rowmap + r) : r;
    for (int j = threadIdx.x; j < cols; j += blockDim.x) {
      const float x = __ldg(in + rin * ld_in + j);
      if (scatter) row[__ldg(colmap + j)] = x; else row[j] = x;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < cols; j += blockDim.x)
      out[r * ld_out + j] = scatter ? row[j] : row[__ldg(colmap + j)];
    __syncthreads();
  }
}

// Packed skew parameters -> dense skew blocks (compact storage, replication review "Summary";
// n_elements = b(b-1)/2, "Reproducibility & code").  Block z, entry (i, j):
//   S = theta[p(i,j)] above the diagonal, -theta[p(j,i)] below, 0 (+1 if add_identity) on it.
// Up to two typed outputs (element (z*b+i, j) at o[(z*b+i)*ld + j]) and one contiguous f32 one.
__global__ void unpack_skew_kernel(const float* __restrict__ theta, long nblocks, int b, void* o1, int dt1,
                                   long ld1, void* o2, int dt2, long ld2, float* of32, int add_identity) {
  sm100::griddep_wait();
  const long bb = (long)b * b;
  const long total = nblocks * bb;
  const long P = (long)b * (b - 1) / 2;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const long z = idx / bb;
    const int rem = (int)(idx - z * bb);
    const int i = rem / b, j = rem - (rem / b) * b;
    float v = 0.f;
    if (i < j) v = __ldg(theta + z * P + packed_pos(i, j, b));
    else if (i > j) v = -__ldg(theta + z * P + packed_pos(j, i, b));
    else if (add_identity) v = 1.f;
    const long row = z * b + i;
    if (o1) store_elem(o1, row * ld1 + j, dt1, v);
    if (o2) store_elem(o2, row * ld2 + j, dt2, v);
    if (of32) of32[idx] = v;
  }
}

// Gradient w.r.t. the packed parameters: g[p(i,j)] = GS[i][j] - GS[j][i] (theta enters S with
// +1 above and -1 below the diagonal).  GS is [nblocks, b, b] f32 contiguous.
__global__ void pack_antisym_kernel(const float* __restrict__ GS, long nblocks, int b, float* __restrict__ g) {
  sm100::griddep_wait();
  const long bb = (long)b * b;
  const long total = nblocks * bb;
  const long P = (long)b * (b - 1) / 2;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const long z = idx / bb;
    const int rem = (int)(idx - z * bb);
    const int i = rem / b, j = rem - (rem / b) * b;
    if (i < j) g[z * P + packed_pos(i, j, b)] = GS[idx] - GS[z * bb + (long)j * b + i];
  }
}

// out[r][c] = sum_s part[s][r][c] (f32, contiguous [rows, cols]); optional typed copy out2 with
// row stride ld2.
__global__ void reduce_splits_kernel(const float* __restrict__ part, int splits, long split_stride, long rows,
                                     int cols, float* __restrict__ out, void* out2, int dt2, long ld2) {
  sm100::griddep_wait();
  const long total = rows * cols;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int q = 0; q < splits; ++q) s += part[q * split_stride + idx];
    out[idx] = s;
    if (out2) {
      const long r = idx / cols;
      store_elem(out2, r * ld2 + (idx - r * cols), dt2, s);
    }
  }
}

__global__ void perm_inverse_kernel(const int32_t* __restrict__ perm, int n, int32_t* __restrict__ inv) {
  sm100::griddep_wait();
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < n; j += gridDim.x * blockDim.x) inv[perm[j]] = j;
}

// sigma[i] = inv_old[new[i]]
__global__ void perm_compose_kernel(const int32_t* __restrict__ inv_old, const int32_t* __restrict__ pnew, int n,
                                    int32_t* __restrict__ sigma) {
  sm100::griddep_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) sigma[i] = inv_old[pnew[i]];
}

// ------------------------------------------------------------ POET-XQ weight format
// Per row o of a bf16 W0' [rows, cols] (cols % 8 == 0): s_o = max_i |w| / 127 and
// q[o, i] = round(w / s_o) to nearest, ties to even, clipped to [-127, 127]; a zero row gets
// s_o = 0 and q = 0.  Both decisions are taken in float32 with IEEE division, so the codes are
// a deterministic function of the bf16 input.  One warp per row: the first pass finds the
// absmax, the second (from L2) writes 8 codes per 16-byte load.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t* __restrict__ W, long ld, long rows,
                                                            int cols, int8_t* __restrict__ q, long ldq,
                                                            float* __restrict__ scale) {
  sm100::griddep_wait();
  const int lane = threadIdx.x & 31, chunks = cols / 8;
  for (long r = (long)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += (long)gridDim.x * 8) {
    const uint4* src = reinterpret_cast<const uint4*>(W + r * ld);
    float amax = 0.f;
    for (int c = lane; c < chunks; c += 32) {
      const uint4 u = src[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[t] << 16)), fabsf(__uint_as_float(w[t] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, 127.f);
    if (lane == 0) scale[r] = s;
    uint2* dst = reinterpret_cast<uint2*>(q + r * ldq);
    for (int c = lane; c < chunks; c += 32) {
      const uint4 u = src[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t packed[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float v = __uint_as_float(e & 1 ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
        const int code = s > 0.f ? min(127, max(-127, __float2int_rn(__fdiv_rn(v, s)))) : 0;
        packed[e >> 2] |= (uint32_t)(code & 0xff) << (8 * (e & 3));
      }
      dst[c] = make_uint2(packed[0], packed[1]);
    }
  }
}

// W0'[o, i] = bf16(s_o * q[o, i]) for [rows, cols] (cols % 8 == 0), eight codes per thread step.
__global__ void __launch_bounds__(256) dequantize_rows_kernel(const int8_t* __restrict__ q, long ldq,
                                                              const float* __restrict__ scale, long rows, int cols,
                                                              uint16_t* __restrict__ W, long ld) {
  sm100::griddep_wait();
  const long chunks = cols / 8, total = rows * chunks;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (long)gridDim.x * blockDim.x) {
    const long r = idx / chunks, c = idx - r * chunks;
    const uint2 w = *reinterpret_cast<const uint2*>(q + r * ldq + c * 8);
    *reinterpret_cast<uint4*>(W + r * ld + c * 8) = dequant8_bf16(w, scale[r]);
  }
}

}  // namespace poetx
