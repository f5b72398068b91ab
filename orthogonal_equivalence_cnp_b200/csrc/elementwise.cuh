// Memory-bound kernels of the POET-X layer: permutation of the feature dimension, packed skew
// unpack / packed-gradient pack, split-K reduction, permutation inverse and composition.
#pragma once

#include "common.cuh"

namespace poetx {

// Position of S[i][j] (i < j) in the packed upper triangle, row by row.
__host__ __device__ __forceinline__ long packed_pos(int i, int j, int b) {
  return (long)i * b - (long)i * (i + 1) / 2 + (j - i - 1);
}

// Index-based permutation of the feature (column) dimension of a row-major [rows, cols] array
// (replication review of POET-X, "Summary": permutations applied by index, never as a matmul;
// Table 1 of the paper measures such a kernel).  A block stages `rb` whole rows in shared
// memory with 16-byte coalesced loads, permutes inside shared memory and writes 16-byte
// coalesced stores, so HBM sees one read and one write of each element.  Each thread keeps
// PERM_VPT independent 16-byte loads in flight (registers first, then shared memory), which is
// what it takes to cover HBM latency at ~16 resident warps per SM.
//   gather (scatter == 0): out[r][j] = in[rowmap ? rowmap[r] : r][colmap[j]]
//   scatter (scatter == 1): out[r][colmap[j]] = in[r][j]
// Requires cols % (16 / sizeof(T)) == 0 and 16-byte aligned rows.
constexpr int PERM_VPT = 8;

template <typename T>
__global__ void __launch_bounds__(256)
    permute_cols_kernel(const T* __restrict__ in, long ld_in, T* __restrict__ out, long ld_out, long rows,
                        int cols, const int32_t* __restrict__ colmap, const int32_t* __restrict__ rowmap,
                        int scatter, int rb) {
  extern __shared__ __align__(16) uint8_t smem_perm[];
  T* buf = reinterpret_cast<T*>(smem_perm);
  constexpr int VEC = 16 / sizeof(T);
  const int nvec = cols / VEC;
  const int nthr = blockDim.x;
  for (long r0 = (long)blockIdx.x * rb; r0 < rows; r0 += (long)gridDim.x * rb) {
    const int nr = (int)min((long)rb, rows - r0);
    const int total = nr * nvec;
    // Phase 1: rows -> registers -> shared memory (gather: as is; scatter: permuted).
    for (int base = threadIdx.x; base < total; base += nthr * PERM_VPT) {
      uint4 v[PERM_VPT];
#pragma unroll
      for (int u = 0; u < PERM_VPT; ++u) {
        const int t = base + u * nthr;
        if (t < total) {
          const int rr = t / nvec, c = t - rr * nvec;
          const long rin = (!scatter && rowmap) ? (long)__ldg(rowmap + r0 + rr) : r0 + rr;
          v[u] = __ldg(reinterpret_cast<const uint4*>(in + rin * ld_in) + c);
        }
      }
#pragma unroll
      for (int u = 0; u < PERM_VPT; ++u) {
        const int t = base + u * nthr;
        if (t < total) {
          const int rr = t / nvec, c = t - rr * nvec;
          T* row = buf + (long)rr * cols;
          if (!scatter) {
            reinterpret_cast<uint4*>(row)[c] = v[u];
          } else {
            const T* vals = reinterpret_cast<const T*>(&v[u]);
            int idx[VEC];
#pragma unroll
            for (int q = 0; q < VEC; q += 4) {
              const int4 m4 = __ldg(reinterpret_cast<const int4*>(colmap + c * VEC + q));
              idx[q] = m4.x; idx[q + 1] = m4.y; idx[q + 2] = m4.z; idx[q + 3] = m4.w;
            }
#pragma unroll
            for (int q = 0; q < VEC; ++q) row[idx[q]] = vals[q];
          }
        }
      }
    }
    __syncthreads();
    // Phase 2: shared memory -> 16-byte coalesced stores (gather: permuted read).
    for (int t = threadIdx.x; t < total; t += nthr) {
      const int rr = t / nvec, c = t - rr * nvec;
      const T* row = buf + (long)rr * cols;
      uint4 o;
      if (!scatter) {
        T vals[VEC];
#pragma unroll
        for (int q = 0; q < VEC; q += 4) {
          const int4 m4 = __ldg(reinterpret_cast<const int4*>(colmap + c * VEC + q));
          vals[q] = row[m4.x]; vals[q + 1] = row[m4.y]; vals[q + 2] = row[m4.z]; vals[q + 3] = row[m4.w];
        }
        o = *reinterpret_cast<const uint4*>(vals);
      } else {
        o = reinterpret_cast<const uint4*>(row)[c];
      }
      reinterpret_cast<uint4*>(out + (r0 + rr) * ld_out)[c] = o;
    }
    __syncthreads();
  }
}

// Packed skew parameters -> dense skew blocks (compact storage, replication review "Summary";
// n_elements = b(b-1)/2, "Reproducibility & code").  Block z, entry (i, j):
//   S = theta[p(i,j)] above the diagonal, -theta[p(j,i)] below, 0 (+1 if add_identity) on it.
// Up to two typed outputs (element (z*b+i, j) at o[(z*b+i)*ld + j]) and one contiguous f32 one.
__global__ void unpack_skew_kernel(const float* __restrict__ theta, long nblocks, int b, void* o1, int dt1,
                                   long ld1, void* o2, int dt2, long ld2, float* of32, int add_identity) {
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
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < n; j += gridDim.x * blockDim.x) inv[perm[j]] = j;
}

// sigma[i] = inv_old[new[i]]
__global__ void perm_compose_kernel(const int32_t* __restrict__ inv_old, const int32_t* __restrict__ pnew, int n,
                                    int32_t* __restrict__ sigma) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) sigma[i] = inv_old[pnew[i]];
}

}  // namespace poetx
