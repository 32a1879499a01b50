// Run-time activation rotate + quantise.
//
// For every token row m and rotation block B:
//     x'_B = H_b . (R_SVD,B^T . x[m, perm[B*b .. B*b+b)])        (fp32)
// i.e. the row form of x' = R^T P^T x with R = blockdiag(R_SVD,B . H_b)
// ("{Omega}-QVLA: Robust Quantization ...", Methodology 1: composite
// SVD.Hadamard rotation applied in blocks after the zigzag permutation).
// Scale selection ("Methodology 2", per-step DiT activation scale table;
// "FoldQuantVLA", dynamic per-token quantisation):
//     DYNAMIC  s = fp32(max_k |x'[m,k]| / 7) over the whole rotated row
//     TABLE    s = table[step][layer], step read on the device
// Codes q = clamp(rint(x'/s), -8, 7) (IEEE fp32 division, ties to even),
// nibble-packed two per byte, even index in the low nibble.
//
// One CTA owns a tile of TT tokens and a contiguous run of rotation blocks.
// Per block it
//   1. gathers x[m, perm[B*b + i]] for its tokens into shared memory (fp32,
//      token-contiguous), while R_SVD,B streams in through cp.async in
//      double-buffered chunks of rows;
//   2. forms R_SVD,B^T x_B with fp32 FMAs in input order, each thread holding a
//      2-channel x TPT-token register tile;
//   3. applies the Walsh-Hadamard factor per token in one warp (butterflies with
//      distance < 32 through shuffles, larger ones in registers) and the
//      1/sqrt(b) scale.
// TABLE mode quantises each block at once.  DYNAMIC mode keeps the CTA's
// rotated slice in shared memory, takes the row maximum across the CTAs of a
// thread-block cluster (the blocks of a row are split over up to 16 CTAs)
// through distributed shared memory, then quantises the kept slice: one pass,
// no scratch memory.
//
// Programmatic dependent launch: the permutation slice and the first R_SVD
// chunk are staged before waiting on the previous kernel in the stream.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "qvla_common.cuh"
#include "qvla_internal.h"

namespace qvla {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemCap = 220 * 1024;

enum Mode { kTable = 0, kDynamic = 1, kRotateOnly = 2 };

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

template <int BS>
struct Geo {
  static constexpr int RCH = BS * BS * 4 <= 32768 ? BS : 8192 / BS;   // R rows per chunk
  static constexpr int NCH = BS / RCH;                                  // chunks per block
  static constexpr int kChunkFloats = RCH * BS;
  static constexpr int NJP = BS / 2;                                    // channel pairs
  static constexpr int NTG = kThreads / NJP;                            // token groups
};

template <int BS, int TT>
struct Smem {
  // [perm slice][R chunk x2][xg / ys][keep]
  static size_t bytes(int nbc, bool keep) {
    size_t b = static_cast<size_t>(nbc) * BS * 4;
    b = (b + 15) & ~static_cast<size_t>(15);
    b += 2 * static_cast<size_t>(Geo<BS>::kChunkFloats) * 4;
    b += static_cast<size_t>(BS) * TT * 4;
    if (keep) b += static_cast<size_t>(TT) * (nbc * BS + 4) * 4;
    return b;
  }
};

QVLA_DEVICE void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
QVLA_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
QVLA_DEVICE void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

QVLA_DEVICE int quant_code(float v, float s, int qmin, int qmax) {
  if (s == 0.f) return 0;
  float r = rintf(__fdiv_rn(v, s));
  r = fminf(fmaxf(r, static_cast<float>(qmin)), static_cast<float>(qmax));
  return static_cast<int>(r);
}

QVLA_DEVICE float load_x(const float* p) { return __ldg(p); }
QVLA_DEVICE float load_x(const __nv_bfloat16* p) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(p)))
                         << 16);
}

// Resolves the table scale; flags the error word and returns 0 when the step
// or layer lies outside the table (never reads outside it).
QVLA_DEVICE float table_scale(const float* table, int T, int Lcount, const int32_t* step_dev,
                              int step_host, int layer, unsigned int* err) {
  const int step = step_dev ? *step_dev : step_host;
  if (step < 0 || step >= T || layer < 0 || layer >= Lcount) {
    report(err, QVLA_DEVERR_STEP_RANGE);
    return 0.f;
  }
  return __ldg(table + static_cast<size_t>(step) * Lcount + layer);
}

template <int BS>
QVLA_DEVICE void fwht_lanes(float (&v)[BS / 32], int lane) {
  constexpr int C = BS / 32;
#pragma unroll
  for (int h = 1; h < 32 && h < BS; h <<= 1) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const float o = __shfl_xor_sync(0xffffffffu, v[c], h);
      v[c] = (lane & h) ? (o - v[c]) : (v[c] + o);
    }
  }
#pragma unroll
  for (int hc = 1; hc < C; hc <<= 1) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
      if ((c & hc) == 0) {
        const float a = v[c], b = v[c | hc];
        v[c] = a + b;
        v[c | hc] = a - b;
      }
    }
  }
#pragma unroll
  for (int c = 0; c < C; ++c) v[c] *= InvSqrtB<BS>::v;
}

// Packs the codes of 32 consecutive channels (lane l holds channel l) into 16
// bytes and stores them as four 32-bit words from lanes 0, 8, 16, 24.
QVLA_DEVICE void store_codes32(uint8_t* dst, int q, int lane) {
  const int qn = __shfl_down_sync(0xffffffffu, q, 1);
  const uint32_t byte = static_cast<uint32_t>((q & 15) | ((qn & 15) << 4));   // even lanes
  const uint32_t b1 = __shfl_down_sync(0xffffffffu, byte, 2);
  const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 4);
  const uint32_t b3 = __shfl_down_sync(0xffffffffu, byte, 6);
  if ((lane & 7) == 0)
    *reinterpret_cast<uint32_t*>(dst + (lane >> 1)) = byte | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

// One linear of a batched launch; CTAs are numbered problem by problem along
// grid x (token tile fastest, then block group); DYNAMIC mode splits each row
// over the cluster along grid y instead.
constexpr int kMaxBatch = 16;
struct ActProblem {
  const void* x;
  const int32_t* perm;
  const float* rot;
  const float* table;
  const int32_t* step_dev;
  uint8_t* xq;
  float* s_x;
  float* xr_out;
  int M, ldx, K, T, Lcount, step_host, layer;
  int gx;                     // token tiles
  int bpc;                    // rotation blocks per CTA
};
struct ActBatch {
  int n;
  int cta_start[kMaxBatch + 1];
  ActProblem p[kMaxBatch];
};

template <int BS, int TT, typename Tin, int MODE>
__global__ void __launch_bounds__(kThreads)
    rotq_kernel(const __grid_constant__ ActBatch batch, unsigned int* err) {
  using G = Geo<BS>;
  constexpr int C = BS / 32;
  constexpr int TPT = TT / G::NTG;          // tokens per thread in the product
  static_assert(TPT >= 1, "token tile too small for this block size");
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ unsigned int amax_s[TT];
  __shared__ float scale_s[TT];

  int pi = 0;
  while (pi + 1 < batch.n && static_cast<int>(blockIdx.x) >= batch.cta_start[pi + 1]) ++pi;
  const ActProblem& P = batch.p[pi];
  const Tin* __restrict__ x = static_cast<const Tin*>(P.x);
  const int M = P.M, ldx = P.ldx, K = P.K;
  const int32_t* __restrict__ perm = P.perm;
  const float* __restrict__ rot = P.rot;
  uint8_t* __restrict__ xq = P.xq;
  float* __restrict__ s_x = P.s_x;
  float* __restrict__ xr_out = P.xr_out;
  const int blocks_per_cta = P.bpc;
  const int local = static_cast<int>(blockIdx.x) - batch.cta_start[pi];
  const int tile = local % P.gx;
  const int group = MODE == kDynamic ? static_cast<int>(blockIdx.y) : local / P.gx;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int m0 = tile * TT;
  const int ntok = min(TT, M - m0);
  const int nb = K / BS;
  const int B0 = group * blocks_per_cta;
  const int nbc = max(0, min(blocks_per_cta, nb - B0));

  int32_t* perm_s = reinterpret_cast<int32_t*>(smem);
  float* rbuf = reinterpret_cast<float*>(
      smem + ((static_cast<size_t>(blocks_per_cta) * BS * 4 + 15) & ~static_cast<size_t>(15)));
  float* xg = rbuf + 2 * G::kChunkFloats;     // [BS][TT], later ys [TT][BS]
  float* keep = xg + BS * TT;                  // [TT][blocks_per_cta*BS + 4]  (DYNAMIC only)
  const int kpitch = blocks_per_cta * BS + 4;

  // ---- prologue: weight-side data, independent of the previous kernel
  for (int e = tid; e < nbc * BS; e += kThreads) perm_s[e] = __ldg(perm + B0 * BS + e);
  if (tid < TT) amax_s[tid] = 0u;
  const int nchunks = nbc * G::NCH;
  auto issue_chunk = [&](int g) {
    const int bl = g / G::NCH, ch = g % G::NCH;
    const float* src = rot + (static_cast<size_t>(B0 + bl) * BS + ch * G::RCH) * BS;
    float* dst = rbuf + (g & 1) * G::kChunkFloats;
    for (int e = tid * 4; e < G::kChunkFloats; e += kThreads * 4) cp_async16(dst + e, src + e);
    cp_async_commit();
  };
  if (nchunks > 0) issue_chunk(0);

  pdl_wait();
  pdl_launch_dependents();
  float s_tab = 0.f;
  if (MODE == kTable)
    s_tab = table_scale(P.table, P.T, P.Lcount, P.step_dev, P.step_host, P.layer, err);
  __syncthreads();   // perm_s visible

  const int jp = tid % G::NJP, tg = tid / G::NJP;
  for (int bl = 0; bl < nbc; ++bl) {
    const int B = B0 + bl;
    // 1. gather the block's inputs, token-contiguous
    for (int e = tid; e < BS * TT; e += kThreads) {
      const int i = e / TT, t = e % TT;
      const int p = perm_s[bl * BS + i];
      float v = 0.f;
      if (t < ntok && static_cast<unsigned>(p) < static_cast<unsigned>(K))
        v = load_x(x + static_cast<size_t>(m0 + t) * ldx + p);
      xg[e] = v;
    }
    // 2. dense product over R chunks
    float acc[TPT][2];
#pragma unroll
    for (int u = 0; u < TPT; ++u) acc[u][0] = acc[u][1] = 0.f;
    for (int ch = 0; ch < G::NCH; ++ch) {
      const int g = bl * G::NCH + ch;
      if (g + 1 < nchunks) {
        issue_chunk(g + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const float* Rc = rbuf + (g & 1) * G::kChunkFloats;
#pragma unroll 4
      for (int ii = 0; ii < G::RCH; ++ii) {
        const float2 r = *reinterpret_cast<const float2*>(Rc + ii * BS + 2 * jp);
        const float* xrow = xg + (ch * G::RCH + ii) * TT + tg * TPT;
#pragma unroll
        for (int u = 0; u < TPT; ++u) {
          const float xv = xrow[u];
          acc[u][0] = fmaf(r.x, xv, acc[u][0]);
          acc[u][1] = fmaf(r.y, xv, acc[u][1]);
        }
      }
      __syncthreads();   // chunk buffer (g & 1) may be refilled next
    }
    // 3. stage the products token-major (over the gather buffer)
#pragma unroll
    for (int u = 0; u < TPT; ++u)
      *reinterpret_cast<float2*>(xg + (tg * TPT + u) * BS + 2 * jp) =
          make_float2(acc[u][0], acc[u][1]);
    __syncthreads();
    // 4. Hadamard factor per token, then quantise / keep / store
    for (int t = warp; t < ntok; t += kWarps) {
      float v[C];
#pragma unroll
      for (int c = 0; c < C; ++c) v[c] = xg[t * BS + lane + 32 * c];
      fwht_lanes<BS>(v, lane);
      if (MODE == kRotateOnly) {
        float* dst = xr_out + static_cast<size_t>(m0 + t) * K + B * BS + lane;
#pragma unroll
        for (int c = 0; c < C; ++c) dst[32 * c] = v[c];
      } else if (MODE == kTable) {
        uint8_t* dst = xq + static_cast<size_t>(m0 + t) * (K / 2) + (B * BS) / 2;
#pragma unroll
        for (int c = 0; c < C; ++c)
          store_codes32(dst + 16 * c, quant_code(v[c], s_tab, -8, 7), lane);
      } else {
        float mx = 0.f;
#pragma unroll
        for (int c = 0; c < C; ++c) {
          keep[t * kpitch + bl * BS + lane + 32 * c] = v[c];
          mx = fmaxf(mx, fabsf(v[c]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) atomicMax(&amax_s[t], __float_as_uint(mx));
      }
    }
    __syncthreads();   // gather buffer reused by the next block
  }

  if (MODE == kTable) {
    if (group == 0 && tid < ntok) s_x[m0 + tid] = s_tab;
    return;
  }
  if (MODE == kRotateOnly) return;

  // ---- DYNAMIC: row maximum over the cluster, then quantise the kept slice
  const int cs = gridDim.y;                    // the cluster spans grid y
  if (cs > 1) {
    cluster_sync();                            // partial maxima published
    if (tid < TT) {
      unsigned int mx = 0u;
      const uint32_t a = smem_u32(&amax_s[tid]);
      for (int r = 0; r < cs; ++r) {
        uint32_t v;
        asm volatile("ld.shared::cluster.u32 %0, [%1];"
                     : "=r"(v)
                     : "r"(map_shared_rank(a, static_cast<uint32_t>(r)))
                     : "memory");
        mx = max(mx, v);
      }
      scale_s[tid] = __fdiv_rn(__uint_as_float(mx), 7.0f);
    }
    cluster_arrive_relaxed();                  // done reading peers' maxima
  } else if (tid < TT) {
    scale_s[tid] = __fdiv_rn(__uint_as_float(amax_s[tid]), 7.0f);
  }
  __syncthreads();
  if (blockIdx.y == 0 && tid < ntok) s_x[m0 + tid] = scale_s[tid];
  const int nch = nbc * BS;                    // channels held by this CTA (multiple of 32)
  for (int t = warp; t < ntok; t += kWarps) {
    const float s = scale_s[t];
    uint8_t* dst = xq + static_cast<size_t>(m0 + t) * (K / 2) + (B0 * BS) / 2;
    for (int c0 = 0; c0 < nch; c0 += 256) {
      const int k = c0 + 8 * lane;            // 8 channels -> 4 bytes per lane
      if (k < nch) {
        const float4 a = *reinterpret_cast<const float4*>(keep + t * kpitch + k);
        const float4 b = *reinterpret_cast<const float4*>(keep + t * kpitch + k + 4);
        const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t w = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int lo = quant_code(f[2 * q], s, -8, 7), hi = quant_code(f[2 * q + 1], s, -8, 7);
          w |= static_cast<uint32_t>((lo & 15) | ((hi & 15) << 4)) << (8 * q);
        }
        *reinterpret_cast<uint32_t*>(dst + k / 2) = w;
      }
    }
  }
  if (cs > 1) cluster_wait();                  // peers finished reading our maxima
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
    s_sh = table_scale(table, T, Lcount, step_dev, step_host, layer, err);
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

// Grid of one problem: token tiles gx, CTAs per token tile (block groups, or
// the cluster size in DYNAMIC mode) and rotation blocks per CTA.
template <int BS, int TT, int MODE>
void problem_grid(int M, int K, int* gx, int* per_tile, int* bpc) {
  const int nb = K / BS;
  *gx = (M + TT - 1) / TT;
  if (MODE == kDynamic) {
    int cs = 1;
    while (cs < 16 && cs < nb &&
           (*gx * cs < 148 || Smem<BS, TT>::bytes((nb + cs - 1) / cs, true) > kSmemCap))
      cs *= 2;
    *bpc = (nb + cs - 1) / cs;
    *per_tile = cs;
  } else {
    const int target = 2 * 148;
    int g = (target + *gx - 1) / *gx;
    g = g < 1 ? 1 : (g > nb ? nb : g);
    *bpc = (nb + g - 1) / g;
    *per_tile = (nb + *bpc - 1) / *bpc;
  }
}

// Launches up to kMaxBatch problems that share (BS, TT, Tin, MODE) and, in
// DYNAMIC mode, the cluster size.
template <int BS, int TT, typename Tin, int MODE>
cudaError_t launch_group(const ActArgs* const* as, int n, cudaStream_t stream) {
  ActBatch batch;
  std::memset(&batch, 0, sizeof(batch));
  batch.n = n;
  int ctas = 0, cs = 1, bpc_max = 1;
  for (int i = 0; i < n; ++i) {
    const ActArgs& a = *as[i];
    int gx, per_tile, bpc;
    problem_grid<BS, TT, MODE>(a.M, a.K, &gx, &per_tile, &bpc);
    ActProblem& P = batch.p[i];
    P.x = a.x;
    P.perm = a.perm;
    P.rot = a.rot;
    P.table = a.table;
    P.step_dev = a.step_dev;
    P.xq = a.xq;
    P.s_x = a.s_x;
    P.xr_out = a.xr_out;
    P.M = a.M;
    P.ldx = a.ldx;
    P.K = a.K;
    P.T = a.T;
    P.Lcount = a.Lcount;
    P.step_host = a.step_host;
    P.layer = a.layer;
    P.gx = gx;
    P.bpc = bpc;
    batch.cta_start[i] = ctas;
    if (MODE == kDynamic) {
      ctas += gx;
      cs = per_tile;                 // equal within a group (the caller groups by it)
    } else {
      ctas += gx * per_tile;
    }
    bpc_max = std::max(bpc_max, bpc);
  }
  batch.cta_start[n] = ctas;
  const size_t smem = Smem<BS, TT>::bytes(bpc_max, MODE == kDynamic);
  if (smem > static_cast<size_t>(kSmemCap)) return cudaErrorInvalidConfiguration;
  auto kern = rotq_kernel<BS, TT, Tin, MODE>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
    if (e != cudaSuccess) return e;
    if (MODE == kDynamic) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas, MODE == kDynamic ? cs : 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (MODE == kDynamic && cs > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = cs;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, batch, device_error_word());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int BS, int TT, typename Tin, int MODE>
cudaError_t launch_cfg_batches(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  if (MODE != kDynamic) {
    for (size_t i0 = 0; i0 < v.size(); i0 += kMaxBatch) {
      const int n = static_cast<int>(std::min<size_t>(kMaxBatch, v.size() - i0));
      cudaError_t e = launch_group<BS, TT, Tin, MODE>(v.data() + i0, n, stream);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  // DYNAMIC: one launch per cluster size
  for (int cs = 1; cs <= 16; cs *= 2) {
    std::vector<const ActArgs*> g;
    for (const ActArgs* a : v) {
      int gx, per_tile, bpc;
      problem_grid<BS, TT, MODE>(a->M, a->K, &gx, &per_tile, &bpc);
      if (per_tile == cs) g.push_back(a);
    }
    for (size_t i0 = 0; i0 < g.size(); i0 += kMaxBatch) {
      const int n = static_cast<int>(std::min<size_t>(kMaxBatch, g.size() - i0));
      cudaError_t e = launch_group<BS, TT, Tin, MODE>(g.data() + i0, n, stream);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

int token_tile_for(int M, int K, int BS, int mode) {
  // 16 for small M, block 32 or very long dynamic rows (keeps the dynamic
  // slice in shared memory), else 32
  return (M <= 16 || BS == 32 || (mode == kDynamic && K > 8192)) ? 16 : 32;
}

template <int BS, typename Tin, int MODE>
cudaError_t launch_bs(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  std::vector<const ActArgs*> t16, t32;
  for (const ActArgs* a : v) (token_tile_for(a->M, a->K, BS, MODE) == 16 ? t16 : t32).push_back(a);
  cudaError_t e = cudaSuccess;
  if (!t16.empty()) e = launch_cfg_batches<BS, 16, Tin, MODE>(t16, stream);
  if (e == cudaSuccess && !t32.empty()) e = launch_cfg_batches<BS, (BS == 32 ? 16 : 32), Tin, MODE>(t32, stream);
  return e;
}

template <typename Tin, int MODE>
cudaError_t launch_mode(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  static const int kBlocks[4] = {32, 64, 128, 256};
  for (int b : kBlocks) {
    std::vector<const ActArgs*> g;
    for (const ActArgs* a : v)
      if (a->block == b) g.push_back(a);
    if (g.empty()) continue;
    cudaError_t e;
    switch (b) {
      case 32: e = launch_bs<32, Tin, MODE>(g, stream); break;
      case 64: e = launch_bs<64, Tin, MODE>(g, stream); break;
      case 128: e = launch_bs<128, Tin, MODE>(g, stream); break;
      default: e = launch_bs<256, Tin, MODE>(g, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename Tin>
cudaError_t launch_dtype(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  std::vector<const ActArgs*> rot, dyn, tab;
  for (const ActArgs* a : v) (a->xq == nullptr ? rot : a->dynamic ? dyn : tab).push_back(a);
  cudaError_t e = cudaSuccess;
  if (!rot.empty()) e = launch_mode<Tin, kRotateOnly>(rot, stream);
  if (e == cudaSuccess && !dyn.empty()) e = launch_mode<Tin, kDynamic>(dyn, stream);
  if (e == cudaSuccess && !tab.empty()) e = launch_mode<Tin, kTable>(tab, stream);
  return e;
}

}  // namespace

cudaError_t launch_rotate_quant_batch(const ActArgs* as, int n, cudaStream_t stream) {
  std::vector<const ActArgs*> bf, f32;
  for (int i = 0; i < n; ++i)
    if (as[i].M > 0) (as[i].xdt == QVLA_DTYPE_BF16 ? bf : f32).push_back(&as[i]);
  cudaError_t e = cudaSuccess;
  if (!bf.empty()) e = launch_dtype<__nv_bfloat16>(bf, stream);
  if (e == cudaSuccess && !f32.empty()) e = launch_dtype<float>(f32, stream);
  return e;
}

cudaError_t launch_rotate_quant(const ActArgs& a, cudaStream_t stream) {
  return launch_rotate_quant_batch(&a, 1, stream);
}

cudaError_t launch_quant_rows(const QuantArgs& a, cudaStream_t stream) {
  quant_rows_kernel<<<a.rows, kThreads, 0, stream>>>(a.xr, a.K, a.qmin, a.qmax, a.dynamic,
                                                     a.table, a.T, a.Lcount, a.step_dev,
                                                     a.step_host, a.layer, a.q_out, a.s_out,
                                                     device_error_word());
  return cudaGetLastError();
}

}  // namespace qvla
