// Offline pack kernels (fp64 on the device):
//  * weight-column L2 norms, the key of the zigzag permutation;
//  * per-block Gram matrices G_B = A_B^T A_B with A_B = (W P)[:, B], whose
//    eigenvectors are the right singular vectors R_SVD,B;
//  * the weight rotation W' = W P R with R_B = R_SVD,B . H_b, formed as a
//    dense fp64 product followed by an fp64 Walsh-Hadamard transform and
//    rounded once to fp32.
// ("{Omega}-QVLA: Robust Quantization ...", Methodology 1: SVD rotation from
// W = U S V^T, normalised Hadamard, block implementation with a zigzag
// permutation by weight-column norm.)
#include <cuda_bf16.h>

#include "qvla_common.cuh"
#include "qvla_internal.h"

namespace qvla {
namespace {

__global__ void column_norms_kernel(const float* __restrict__ W, int N, int K,
                                    double* __restrict__ norms) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double s = 0.0;
  for (int n = 0; n < N; ++n) {
    const double w = static_cast<double>(__ldg(W + static_cast<size_t>(n) * K + k));
    s = fma(w, w, s);
  }
  norms[k] = sqrt(s);
}

// Gram tile of one block: G_B[i0 + i][j0 + j], TS x TS entries per CTA.
template <int TS>
__global__ void __launch_bounds__(256)
    block_gram_kernel(const float* __restrict__ W, int N, int K, int block,
                      const int32_t* __restrict__ perm, double* __restrict__ gram) {
  constexpr int RN = 32;                 // rows of W per smem chunk
  constexpr int PT = TS * TS / 256;      // entries per thread
  constexpr int SIDE = TS / 16;          // per-thread register tile side (PT = SIDE^2)
  __shared__ double Ai[RN][TS];
  __shared__ double Aj[RN][TS];
  const int B = blockIdx.x;
  const int tiles = block / TS;
  const int i0 = (blockIdx.y / tiles) * TS, j0 = (blockIdx.y % tiles) * TS;
  const int tid = threadIdx.x;
  const int ti = (tid / 16) * SIDE, tj = (tid % 16) * SIDE;
  const int32_t* pB = perm + static_cast<size_t>(B) * block;
  double acc[SIDE][SIDE];
#pragma unroll
  for (int a = 0; a < SIDE; ++a)
#pragma unroll
    for (int b = 0; b < SIDE; ++b) acc[a][b] = 0.0;
  for (int n0 = 0; n0 < N; n0 += RN) {
    for (int e = tid; e < RN * TS; e += 256) {
      const int r = e / TS, c = e % TS;
      const int n = n0 + r;
      double vi = 0.0, vj = 0.0;
      if (n < N) {
        vi = static_cast<double>(W[static_cast<size_t>(n) * K + pB[i0 + c]]);
        vj = static_cast<double>(W[static_cast<size_t>(n) * K + pB[j0 + c]]);
      }
      Ai[r][c] = vi;
      Aj[r][c] = vj;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < RN; ++r) {
      double a[SIDE], b[SIDE];
#pragma unroll
      for (int u = 0; u < SIDE; ++u) {
        a[u] = Ai[r][ti + u];
        b[u] = Aj[r][tj + u];
      }
#pragma unroll
      for (int u = 0; u < SIDE; ++u)
#pragma unroll
        for (int v = 0; v < SIDE; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
  (void)PT;
  double* G = gram + static_cast<size_t>(B) * block * block;
#pragma unroll
  for (int u = 0; u < SIDE; ++u)
#pragma unroll
    for (int v = 0; v < SIDE; ++v)
      G[static_cast<size_t>(i0 + ti + u) * block + (j0 + tj + v)] = acc[u][v];
}

// W'[n, B*BS + j] = fp32( sum_i W[n, perm[B*BS+i]] (R_SVD,B H_b)[i][j] ) for 8
// rows per CTA (one warp per row); lane l holds columns l + 32c.
template <int BS>
__global__ void __launch_bounds__(256)
    rotate_weights_kernel(const float* __restrict__ W, int N, int K,
                          const int32_t* __restrict__ perm, const double* __restrict__ rsvd,
                          float* __restrict__ Wr) {
  constexpr int C = BS / 32;
  __shared__ double A[8][BS];
  const int B = blockIdx.y;
  const int n0 = blockIdx.x * 8;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* pB = perm + static_cast<size_t>(B) * BS;
  for (int e = tid; e < 8 * BS; e += 256) {
    const int r = e / BS, i = e % BS;
    const int n = n0 + r;
    A[r][i] = n < N ? static_cast<double>(W[static_cast<size_t>(n) * K + pB[i]]) : 0.0;
  }
  __syncthreads();
  const int n = n0 + warp;
  if (n >= N) return;
  const double* R = rsvd + static_cast<size_t>(B) * BS * BS;
  double acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.0;
  for (int i = 0; i < BS; ++i) {
    const double a = A[warp][i];
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = fma(a, R[i * BS + lane + 32 * c], acc[c]);
  }
#pragma unroll
  for (int h = 1; h < 32 && h < BS; h <<= 1) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const double o = __shfl_xor_sync(0xffffffffu, acc[c], h);
      acc[c] = (lane & h) ? (o - acc[c]) : (acc[c] + o);
    }
  }
#pragma unroll
  for (int hc = 1; hc < C; hc <<= 1) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
      if ((c & hc) == 0) {
        const double a = acc[c], b = acc[c | hc];
        acc[c] = a + b;
        acc[c | hc] = a - b;
      }
    }
  }
  const double inv = 1.0 / sqrt(static_cast<double>(BS));
  float* dst = Wr + static_cast<size_t>(n) * K + static_cast<size_t>(B) * BS + lane;
#pragma unroll
  for (int c = 0; c < C; ++c) dst[32 * c] = static_cast<float>(acc[c] * inv);
}

// Tensor-core image of the composite rotation: R_B = R_SVD,B . H_b in fp64,
// split into bf16 parts hi + mid + lo (each the round-to-nearest bf16 of what
// the previous parts leave), stored as R_B^T rows in the 128-byte-swizzled
// K-major layout (see qvla.h).  One thread per element (i, j) of R_B.
template <int BS>
__global__ void __launch_bounds__(256)
    rot_tc_image_kernel(const double* __restrict__ rsvd, uint16_t* __restrict__ img) {
  const int B = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= BS * BS) return;
  const int i = e / BS, j = e % BS;           // R_B[i][j]: input i, output j
  const double* R = rsvd + static_cast<size_t>(B) * BS * BS;
  const double inv = 1.0 / sqrt(static_cast<double>(BS));
  double v = 0.0;
  for (int k = 0; k < BS; ++k) {
    const double h = (__popc(k & j) & 1) ? -inv : inv;
    v = fma(R[i * BS + k], h, v);
  }
  uint16_t* base = img + static_cast<size_t>(B) * 3 * BS * BS;
  const int kc = i / 64, c = (i % 64) / 8;
  const size_t off = static_cast<size_t>(kc) * BS * 64 + j * 64 + ((c ^ (j & 7)) * 8) + (i % 8);
  double r = v;
#pragma unroll
  for (int sp = 0; sp < 3; ++sp) {
    const __nv_bfloat16 part = __double2bfloat16(r);
    r -= static_cast<double>(__bfloat162float(part));
    base[static_cast<size_t>(sp) * BS * BS + off] = __bfloat16_as_ushort(part);
  }
}

}  // namespace

cudaError_t launch_rot_tc_image(const double* rsvd64, int K, int block, uint16_t* img,
                                cudaStream_t s) {
  const int nb = K / block;
  const dim3 grid((block * block + 255) / 256, nb);
  if (block == 64) {
    rot_tc_image_kernel<64><<<grid, 256, 0, s>>>(rsvd64, img);
  } else if (block == 128) {
    rot_tc_image_kernel<128><<<grid, 256, 0, s>>>(rsvd64, img);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_column_norms(const float* W, int N, int K, double* norms, cudaStream_t s) {
  column_norms_kernel<<<(K + 255) / 256, 256, 0, s>>>(W, N, K, norms);
  return cudaGetLastError();
}

cudaError_t launch_block_gram(const float* W, int N, int K, int block, const int32_t* perm,
                              double* gram, cudaStream_t s) {
  const int nb = K / block;
  if (block == 32) {
    block_gram_kernel<32><<<dim3(nb, 1), 256, 0, s>>>(W, N, K, block, perm, gram);
  } else {
    const int tiles = block / 64;
    block_gram_kernel<64><<<dim3(nb, tiles * tiles), 256, 0, s>>>(W, N, K, block, perm, gram);
  }
  return cudaGetLastError();
}

cudaError_t launch_rotate_weights(const float* W, int N, int K, int block, const int32_t* perm,
                                  const double* rsvd64, float* Wr, cudaStream_t s) {
  const dim3 grid((N + 7) / 8, K / block);
  switch (block) {
    case 32: rotate_weights_kernel<32><<<grid, 256, 0, s>>>(W, N, K, perm, rsvd64, Wr); break;
    case 64: rotate_weights_kernel<64><<<grid, 256, 0, s>>>(W, N, K, perm, rsvd64, Wr); break;
    case 128: rotate_weights_kernel<128><<<grid, 256, 0, s>>>(W, N, K, perm, rsvd64, Wr); break;
    case 256: rotate_weights_kernel<256><<<grid, 256, 0, s>>>(W, N, K, perm, rsvd64, Wr); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace qvla
