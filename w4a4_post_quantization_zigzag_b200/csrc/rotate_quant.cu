// Run-time activation rotate + quantise (CUDA-core path).
//
// For every token row m and rotation block B:
//     x'_B = H_b . (R_SVD,B^T . x[m, perm[B*b .. B*b+b)])        (fp32)
// i.e. the row form of x' = R^T P^T x with R = blockdiag(R_SVD,B . H_b)
// ("{Omega}-QVLA: Robust Quantization ...", Methodology 1: composite
// SVD.Hadamard rotation applied in blocks after the zigzag permutation).
// The dense b x b product runs as fp32 FMAs in input order; the Hadamard
// factor is a fast Walsh-Hadamard transform: butterflies with distance < 32
// through warp shuffles, larger distances inside each lane's registers, then
// one multiply by 1/sqrt(b).
//
// Scale selection ("Methodology 2", per-step DiT activation scale table;
// "FoldQuantVLA", dynamic per-token quantisation):
//     DYNAMIC  s = fp32(max_k |x'[m,k]| / 7) over the whole rotated row
//     TABLE    s = table[step][layer], step read on the device
// Codes q = clamp(rint(x'/s), -8, 7) (IEEE fp32 division, ties to even),
// nibble-packed two per byte, even index in the low nibble.
//
// Work split: a CTA stages `tpc` token rows in shared memory (fp32) and its
// warps walk (token, block) items.  DYNAMIC mode keeps whole rows in one CTA
// and recomputes the rotation in a second pass once the row maximum is known
// (no scratch memory, one launch); TABLE mode splits the blocks of a row over
// several CTAs.
#include <cuda_bf16.h>

#include "qvla_common.cuh"
#include "qvla_internal.h"

namespace qvla {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr size_t kRowSmemBudget = 96 * 1024;
constexpr size_t kRowSmemCeiling = QVLA_MAX_K * sizeof(float);   // 128 KB: one row at K max

template <int BS>
struct InvSqrtB;
template <>
struct InvSqrtB<32> {
  static constexpr float v = 0.17677669529663687f;
};
template <>
struct InvSqrtB<64> {
  static constexpr float v = 0.125f;
};
template <>
struct InvSqrtB<128> {
  static constexpr float v = 0.08838834764831845f;
};
template <>
struct InvSqrtB<256> {
  static constexpr float v = 0.0625f;
};

// One warp rotates one block of one token.  On return lane l holds
// v[c] = x'[B*BS + l + 32c].
template <int BS>
QVLA_DEVICE void rotate_block_warp(const float* __restrict__ xs, int K,
                                   const int32_t* __restrict__ permB,
                                   const float* __restrict__ RB, int lane, float (&v)[BS / 32]) {
  constexpr int C = BS / 32;
  float acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.f;
  // (R_SVD,B^T x_B)_j = sum_i R_SVD,B[i][j] * x_B[i]
#pragma unroll 4
  for (int i = 0; i < BS; ++i) {
    const int p = __ldg(permB + i);
    const float xi = xs[static_cast<unsigned>(p) < static_cast<unsigned>(K) ? p : 0];
    const float* Rrow = RB + i * BS + lane;
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = fmaf(__ldg(Rrow + 32 * c), xi, acc[c]);
  }
  // Walsh-Hadamard butterflies; element j = lane + 32c.
#pragma unroll
  for (int h = 1; h < 32 && h < BS; h <<= 1) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const float o = __shfl_xor_sync(0xffffffffu, acc[c], h);
      acc[c] = (lane & h) ? (o - acc[c]) : (acc[c] + o);
    }
  }
#pragma unroll
  for (int hc = 1; hc < C; hc <<= 1) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
      if ((c & hc) == 0) {
        const float a = acc[c], b = acc[c | hc];
        acc[c] = a + b;
        acc[c | hc] = a - b;
      }
    }
  }
#pragma unroll
  for (int c = 0; c < C; ++c) v[c] = acc[c] * InvSqrtB<BS>::v;
}

QVLA_DEVICE int quant_code(float v, float s, int qmin, int qmax) {
  if (s == 0.f) return 0;
  float r = rintf(__fdiv_rn(v, s));
  r = fminf(fmaxf(r, static_cast<float>(qmin)), static_cast<float>(qmax));
  return static_cast<int>(r);
}

template <typename Tin>
QVLA_DEVICE void stage_row(const Tin* __restrict__ src, float* __restrict__ dst, int K, int tid);

template <>
QVLA_DEVICE void stage_row<float>(const float* __restrict__ src, float* __restrict__ dst, int K,
                                  int tid) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
  float4* d4 = reinterpret_cast<float4*>(dst);
  for (int i = tid; i < K / 4; i += kThreads) d4[i] = __ldg(s4 + i);
}

template <>
QVLA_DEVICE void stage_row<__nv_bfloat16>(const __nv_bfloat16* __restrict__ src,
                                          float* __restrict__ dst, int K, int tid) {
  const uint4* s8 = reinterpret_cast<const uint4*>(src);
  for (int i = tid; i < K / 8; i += kThreads) {
    const uint4 u = __ldg(s8 + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float4 lo, hi;
    lo.x = __uint_as_float(w[0] << 16);
    lo.y = __uint_as_float(w[0] & 0xFFFF0000u);
    lo.z = __uint_as_float(w[1] << 16);
    lo.w = __uint_as_float(w[1] & 0xFFFF0000u);
    hi.x = __uint_as_float(w[2] << 16);
    hi.y = __uint_as_float(w[2] & 0xFFFF0000u);
    hi.z = __uint_as_float(w[3] << 16);
    hi.w = __uint_as_float(w[3] & 0xFFFF0000u);
    reinterpret_cast<float4*>(dst)[2 * i] = lo;
    reinterpret_cast<float4*>(dst)[2 * i + 1] = hi;
  }
}

// Resolves the table scale; returns false (and flags the error word) when the
// device step index lies outside the table.
QVLA_DEVICE bool table_scale(const float* table, int T, int Lcount, const int32_t* step_dev,
                             int step_host, int layer, float* s, unsigned int* err) {
  const int step = step_dev ? *step_dev : step_host;
  if (step < 0 || step >= T || layer < 0 || layer >= Lcount) {
    if (threadIdx.x == 0) report(err, QVLA_DEVERR_STEP_RANGE);
    *s = 0.f;
    return false;
  }
  *s = __ldg(table + static_cast<size_t>(step) * Lcount + layer);
  return true;
}

template <int BS, typename Tin, bool kRotateOnly>
__global__ void __launch_bounds__(kThreads)
    rotate_quant_kernel(const Tin* __restrict__ x, int M, int ldx, int K,
                        const int32_t* __restrict__ perm, const float* __restrict__ rot,
                        int dynamic, const float* __restrict__ table, int T, int Lcount,
                        const int32_t* __restrict__ step_dev, int step_host, int layer,
                        uint8_t* __restrict__ xq, float* __restrict__ s_x,
                        float* __restrict__ xr_out, unsigned int* err, int tpc, int bpc) {
  constexpr int C = BS / 32;
  extern __shared__ __align__(16) float smem_rows[];
  __shared__ unsigned int amax_bits[8];
  __shared__ float s_table;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int m0 = blockIdx.x * tpc;
  const int ntok = min(tpc, M - m0);
  const int nb = K / BS;
  const int b0 = blockIdx.y * bpc;
  const int nblk = min(bpc, nb - b0);
  if (ntok <= 0 || nblk <= 0) return;

  for (int t = 0; t < ntok; ++t)
    stage_row<Tin>(x + static_cast<size_t>(m0 + t) * ldx, smem_rows + static_cast<size_t>(t) * K,
                   K, tid);
  if (tid < 8) amax_bits[tid] = 0u;
  if (tid == 0) {
    float s = 0.f;
    if (!kRotateOnly && !dynamic) table_scale(table, T, Lcount, step_dev, step_host, layer, &s, err);
    s_table = s;
  }
  __syncthreads();

  const int nitems = ntok * nblk;
  float v[C];

  if (kRotateOnly) {
    for (int it = warp; it < nitems; it += kWarps) {
      const int t = it / nblk, B = b0 + it % nblk;
      rotate_block_warp<BS>(smem_rows + static_cast<size_t>(t) * K, K, perm + B * BS,
                            rot + static_cast<size_t>(B) * BS * BS, lane, v);
      float* dst = xr_out + static_cast<size_t>(m0 + t) * K + B * BS + lane;
#pragma unroll
      for (int c = 0; c < C; ++c) dst[32 * c] = v[c];
    }
    return;
  }

  if (dynamic) {
    // pass 1: row maxima of |x'|
    for (int it = warp; it < nitems; it += kWarps) {
      const int t = it / nblk, B = b0 + it % nblk;
      rotate_block_warp<BS>(smem_rows + static_cast<size_t>(t) * K, K, perm + B * BS,
                            rot + static_cast<size_t>(B) * BS * BS, lane, v);
      float mx = 0.f;
#pragma unroll
      for (int c = 0; c < C; ++c) mx = fmaxf(mx, fabsf(v[c]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) atomicMax(&amax_bits[t], __float_as_uint(mx));
    }
    __syncthreads();
  }

  // pass 2: quantise and pack
  for (int it = warp; it < nitems; it += kWarps) {
    const int t = it / nblk, B = b0 + it % nblk;
    rotate_block_warp<BS>(smem_rows + static_cast<size_t>(t) * K, K, perm + B * BS,
                          rot + static_cast<size_t>(B) * BS * BS, lane, v);
    const float s = dynamic ? __fdiv_rn(__uint_as_float(amax_bits[t]), 7.0f) : s_table;
    uint8_t* dst = xq + static_cast<size_t>(m0 + t) * (K / 2) + (B * BS) / 2;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int q = quant_code(v[c], s, -8, 7);
      const int qn = __shfl_down_sync(0xffffffffu, q, 1);
      if ((lane & 1) == 0) dst[(lane + 32 * c) >> 1] = static_cast<uint8_t>((q & 15) | ((qn & 15) << 4));
    }
  }

  if (blockIdx.y == 0 && tid < ntok)
    s_x[m0 + tid] = dynamic ? __fdiv_rn(__uint_as_float(amax_bits[tid]), 7.0f) : s_table;
}

// Quantise fp32 rows (already rotated): one CTA per row.
__global__ void __launch_bounds__(kThreads)
    quant_rows_kernel(const float* __restrict__ xr, int K, int qmin, int qmax, int dynamic,
                      const float* __restrict__ table, int T, int Lcount,
                      const int32_t* __restrict__ step_dev, int step_host, int layer,
                      uint8_t* __restrict__ q_out, float* __restrict__ s_out,
                      unsigned int* err) {
  __shared__ float red[kWarps];
  __shared__ float s_sh;
  const int row = blockIdx.x, tid = threadIdx.x;
  const float* src = xr + static_cast<size_t>(row) * K;
  if (dynamic) {
    float mx = 0.f;
    for (int k = tid; k < K; k += kThreads) mx = fmaxf(mx, fabsf(src[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    if (tid == 0) {
      float m = 0.f;
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w]);
      s_sh = __fdiv_rn(m, static_cast<float>(qmax));
    }
  } else if (tid == 0) {
    float s;
    table_scale(table, T, Lcount, step_dev, step_host, layer, &s, err);
    s_sh = s;
  }
  __syncthreads();
  const float s = s_sh;
  uint8_t* dst = q_out + static_cast<size_t>(row) * (K / 2);
  for (int j = tid; j < K / 2; j += kThreads) {
    const int q0 = quant_code(src[2 * j], s, qmin, qmax);
    const int q1 = quant_code(src[2 * j + 1], s, qmin, qmax);
    dst[j] = static_cast<uint8_t>((q0 & 15) | ((q1 & 15) << 4));
  }
  if (tid == 0) s_out[row] = s;
}

template <int BS, typename Tin, bool kRotateOnly>
cudaError_t launch_bs(const ActArgs& a, cudaStream_t stream) {
  const int K = a.K, nb = K / BS;
  int tpc = static_cast<int>(kRowSmemBudget / (static_cast<size_t>(K) * sizeof(float)));
  tpc = tpc < 1 ? 1 : (tpc > 8 ? 8 : tpc);
  const int gx = (a.M + tpc - 1) / tpc;
  int gy = 1;
  if (!a.dynamic || kRotateOnly) {
    const int target = 2 * 148;
    gy = (target + gx - 1) / gx;
    if (gy > nb) gy = nb;
    if (gy < 1) gy = 1;
  }
  const int bpc = (nb + gy - 1) / gy;
  gy = (nb + bpc - 1) / bpc;
  const size_t smem = static_cast<size_t>(tpc) * K * sizeof(float);
  auto kern = rotate_quant_kernel<BS, Tin, kRotateOnly>;
  // one fixed ceiling per kernel (the largest row stage any K can ask for), so
  // launches captured in a graph never see the attribute shrink afterwards
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kRowSmemCeiling));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (smem > kRowSmemCeiling) return cudaErrorInvalidValue;
  kern<<<dim3(gx, gy), kThreads, smem, stream>>>(
      static_cast<const Tin*>(a.x), a.M, a.ldx, K, a.perm, a.rot, a.dynamic, a.table, a.T,
      a.Lcount, a.step_dev, a.step_host, a.layer, a.xq, a.s_x, a.xr_out, device_error_word(),
      tpc, bpc);
  return cudaGetLastError();
}

template <typename Tin, bool kRotateOnly>
cudaError_t launch_t(const ActArgs& a, cudaStream_t stream) {
  switch (a.block) {
    case 32: return launch_bs<32, Tin, kRotateOnly>(a, stream);
    case 64: return launch_bs<64, Tin, kRotateOnly>(a, stream);
    case 128: return launch_bs<128, Tin, kRotateOnly>(a, stream);
    case 256: return launch_bs<256, Tin, kRotateOnly>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_rotate_quant(const ActArgs& a, cudaStream_t stream) {
  const bool rot_only = a.xq == nullptr;
  if (a.xdt == QVLA_DTYPE_BF16)
    return rot_only ? launch_t<__nv_bfloat16, true>(a, stream)
                    : launch_t<__nv_bfloat16, false>(a, stream);
  return rot_only ? launch_t<float, true>(a, stream) : launch_t<float, false>(a, stream);
}

cudaError_t launch_quant_rows(const QuantArgs& a, cudaStream_t stream) {
  quant_rows_kernel<<<a.rows, kThreads, 0, stream>>>(a.xr, a.K, a.qmin, a.qmax, a.dynamic,
                                                     a.table, a.T, a.Lcount, a.step_dev,
                                                     a.step_host, a.layer, a.q_out, a.s_out,
                                                     device_error_word());
  return cudaGetLastError();
}

}  // namespace qvla
