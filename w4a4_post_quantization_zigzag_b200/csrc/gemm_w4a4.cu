// W4A4 GEMM on the sm_100a tensor cores with a fused dequantisation epilogue.
//
//   acc[m,n] = sum_k q_x[m,k] q_w[n,k]                      (exact)
//   y[m,n]   = bf16( fp32(s_x[m] s_w[n]) * acc[m,n] + b[n] )
//
// ("Omega-QVLA: Nen VLA W4A4 tren Edge", section "Vi sao W4A4 kho hon
// W4A16?": weights and activations both 4-bit so the product runs on integer
// tensor cores; "FoldQuantVLA": native integer W4A4 execution.)
//
// sm_100a has no 4-bit integer MMA, so each CTA
//   1. TMA-loads packed int4 tiles (128 bytes of K per row, 128B swizzle) of
//      the weights [128 rows] and the activations [NT rows] into a ring of
//      shared-memory stages (one elected producer thread);
//   2. unpacks them with four warps into the UMMA K-major "interleaved"
//      layout: every code q becomes the int8 value 16*q (its nibble moved into
//      the high half of the byte: `w & 0xF0F0F0F0` for odd codes,
//      `(w << 4) & 0xF0F0F0F0` for even codes).  Even codes of a 32-code
//      group fill the first 16-byte K chunk and odd codes the second; both
//      operands use the same K order, so the dot product is unchanged;
//   3. issues tcgen05.mma kind::i8 (M=128 weight rows, N=NT tokens, K=32)
//      from one thread into an int32 accumulator in tensor memory, which
//      therefore holds 256*acc exactly;
//   4. reads the accumulator back with tcgen05.ld (one output channel per
//      thread, tokens along registers) and applies the epilogue.
// Weights take the UMMA M slot and tokens the N slot for every M, so the small
// token counts of a DiT action chunk (16-64) still fill a 128-row MMA.
// Small M adds split-K over a thread-block cluster along grid z: every CTA of
// the cluster owns a contiguous run of 256-wide K tiles, and the int32 partial
// tiles are summed through distributed shared memory (exact, no workspace).
//
// All waits are bounded (2 s) and flag QVLA_DEVERR_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>

#include "qvla_common.cuh"
#include "qvla_internal.h"

namespace qvla {
namespace {

constexpr int kBM = 128;                  // weight rows per tile (UMMA M)
constexpr int kKP = 256;                  // K per packed stage (128 bytes per row)
constexpr int kKU = 128;                  // K per unpacked stage (128 int8 per row)
constexpr int kRowP = kKP / 2;            // packed bytes per row per stage
constexpr int kThreads = 192;             // warp0 TMA, warp1 MMA, warps2-5 unpack+epilogue
constexpr int kWorkers = 128;

template <int NT>
struct Cfg {
  static constexpr int kRows = kBM + NT;
  static constexpr int kPStageBytes = kRows * kRowP;   // packed: A rows then B rows
  static constexpr int kUStageBytes = kRows * kKU;     // unpacked int8
  static constexpr int kPS = 2;
  static constexpr int kUS = 2;
  static constexpr int kTmemCols = NT < 32 ? 32 : NT;
  static constexpr int kRedPitch = NT + 4;             // int32 per row of the split-K buffer
  static constexpr int kStageBytes = kPS * kPStageBytes + kUS * kUStageBytes;
  static constexpr int kRecvBytes = kBM * kRedPitch * 4;   // split-K receive buffer
  static constexpr int kSmemBytes = kStageBytes + 1024;    // + kRecvBytes when split
  static constexpr bool kCanSplit = kSmemBytes + kRecvBytes <= 227 * 1024;
};

struct Barriers {
  uint64_t full_p[4], empty_p[4], full_u[4], empty_u[4], acc_full;
  uint32_t tmem_base;
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_x, int M, int N, int K,
                     const float* __restrict__ s_x, const float* __restrict__ s_w,
                     const float* __restrict__ bias, __nv_bfloat16* __restrict__ y, int ldy,
                     int32_t* __restrict__ acc_out, unsigned int* err) {
  using C = Cfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Barriers bars;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kBM;
  const int m0 = blockIdx.y * NT;
  const int S = gridDim.z;
  const int split = blockIdx.z;
  const int nkt = (K + kKP - 1) / kKP;
  const int kt0 = split * nkt / S, kt1 = (split + 1) * nkt / S;
  const int nk = kt1 - kt0;

  // 1024-byte aligned stage memory (128B-swizzled TMA destinations)
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* const base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* const pstage = base;
  uint8_t* const ustage = base + C::kPS * C::kPStageBytes;

  if (tid == 0) {
    for (int s = 0; s < C::kPS; ++s) {
      mbar_init(&bars.full_p[s], 1);
      mbar_init(&bars.empty_p[s], kWorkers);
    }
    for (int u = 0; u < C::kUS; ++u) {
      mbar_init(&bars.full_u[u], kWorkers);
      mbar_init(&bars.empty_u[u], 1);
    }
    mbar_init(&bars.acc_full, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_x);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = bars.tmem_base;
  // split-K: announce that this CTA runs; remote shared-memory stores wait for
  // every CTA of the cluster to have done so
  if (S > 1) cluster_arrive_relaxed();
  bool cluster_waited = false;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      // Weights do not depend on the previous kernel in the stream: the first
      // stages' weight tiles are requested before waiting for it (programmatic
      // dependent launch), the activation tiles after.
      const int pre = nk < C::kPS ? nk : C::kPS;
      // the whole weight range of this CTA is requested into L2 at once, so
      // HBM streaming is not limited by the depth of the stage ring
      for (int i = pre; i < nk; ++i) tma_prefetch_l2_2d(&tmap_w, (kt0 + i) * kRowP, n0);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&bars.full_p[i], C::kPStageBytes);
        tma_load_2d(pstage + i * C::kPStageBytes, &tmap_w, &bars.full_p[i], (kt0 + i) * kRowP, n0);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        tma_load_2d(pstage + i * C::kPStageBytes + kBM * kRowP, &tmap_x, &bars.full_p[i],
                    (kt0 + i) * kRowP, m0);
        ++issued;
      }
      for (int i = pre; i < nk && ok; ++i) {
        const int s = i % C::kPS;
        const uint32_t ph = (i / C::kPS) & 1;
        ok = mbar_wait(&bars.empty_p[s], ph ^ 1u, err);
        if (!ok) break;
        uint8_t* dst = pstage + s * C::kPStageBytes;
        mbar_arrive_expect_tx(&bars.full_p[s], C::kPStageBytes);
        const int xbyte = (kt0 + i) * kRowP;
        tma_load_2d(dst, &tmap_w, &bars.full_p[s], xbyte, n0);
        tma_load_2d(dst + kBM * kRowP, &tmap_x, &bars.full_p[s], xbyte, m0);
        ++issued;
      }
      // never leave with copies in flight: wait for the last load of each stage
      for (int i = issued - C::kPS < 0 ? 0 : issued - C::kPS; i < issued; ++i)
        mbar_wait(&bars.full_p[i % C::kPS], (i / C::kPS) & 1, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, NT);
      const uint32_t u_base = smem_u32(ustage);
      bool ok = true;
      for (int j = 0; j < 2 * nk && ok; ++j) {
        const int u = j % C::kUS;
        ok = mbar_wait(&bars.full_u[u], (j / C::kUS) & 1, err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = u_base + u * C::kUStageBytes;
        const uint32_t b0 = a0 + kBM * kKU;
#pragma unroll
        for (int q = 0; q < kKU / 32; ++q) {
          // chunks 2q (even codes) and 2q+1 (odd codes) of this stage
          const uint64_t ad = smem_desc_kmajor_noswizzle(a0 + 2 * q * (kBM * 16), kBM * 16, 128);
          const uint64_t bd = smem_desc_kmajor_noswizzle(b0 + 2 * q * (NT * 16), NT * 16, 128);
          umma_i8(tmem_d, ad, bd, idesc, (j > 0 || q > 0) ? 1u : 0u);
        }
        umma_commit(&bars.empty_u[u]);
      }
      umma_commit(&bars.acc_full);
      mbar_wait(&bars.acc_full, 0, err);   // tensor memory is freed only after this
    }
  } else {
    // --------------------------------------------------- unpack (4 warps)
    const int wt = tid - 64;   // 0..127
    bool ok = true;
    for (int i = 0; i < nk && ok; ++i) {
      const int s = i % C::kPS;
      ok = mbar_wait(&bars.full_p[s], (i / C::kPS) & 1, err);
      if (!ok) break;
      const uint8_t* ps = pstage + s * C::kPStageBytes;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 2 * i + h;
        const int u = j % C::kUS;
        ok = mbar_wait(&bars.empty_u[u], ((j / C::kUS) & 1) ^ 1u, err);
        if (!ok) break;
        uint8_t* us = ustage + u * C::kUStageBytes;
        for (int it = wt; it < C::kRows * 4; it += kWorkers) {
          const bool isA = it < kBM * 4;
          const int e = isA ? it : it - kBM * 4;
          const int r = (e >> 5) * 8 + (e & 7);        // 8 consecutive threads: 8 rows
          const int cl = (e >> 3) & 3;                 // packed 16-byte chunk in this half
          const int rows = isA ? kBM : NT;
          const uint8_t* src = ps + (isA ? 0 : kBM * kRowP) + r * kRowP +
                               ((((4 * h + cl) ^ (r & 7))) << 4);
          const uint4 w = *reinterpret_cast<const uint4*>(src);
          uint4 ev, od;
          ev.x = (w.x << 4) & 0xF0F0F0F0u;
          ev.y = (w.y << 4) & 0xF0F0F0F0u;
          ev.z = (w.z << 4) & 0xF0F0F0F0u;
          ev.w = (w.w << 4) & 0xF0F0F0F0u;
          od.x = w.x & 0xF0F0F0F0u;
          od.y = w.y & 0xF0F0F0F0u;
          od.z = w.z & 0xF0F0F0F0u;
          od.w = w.w & 0xF0F0F0F0u;
          uint8_t* dreg = us + (isA ? 0 : kBM * kKU);
          const int core = (r >> 3) * 128 + (r & 7) * 16;
          *reinterpret_cast<uint4*>(dreg + (2 * cl) * (rows * 16) + core) = ev;
          *reinterpret_cast<uint4*>(dreg + (2 * cl + 1) * (rows * 16) + core) = od;
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars.full_u[u]);
      }
      mbar_arrive(&bars.empty_p[s]);
    }

    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int nl = quarter * 32 + lane;          // local output channel (TMEM lane)
    const int n = n0 + nl;
    const bool have = ok && mbar_wait(&bars.acc_full, 0, err);
    tc_fence_after();
    pdl_launch_dependents();
    pdl_wait();                       // s_x comes from the previous kernel
    if (have) {
      const float sw = (n < N) ? __ldg(s_w + n) : 0.f;
      const float bn = (bias != nullptr && n < N) ? __ldg(bias + n) : 0.f;
      // split-K: this CTA's partial rows go to the receive buffer of the CTA
      // that owns them (rows [r*128/S, (r+1)*128/S) belong to cluster rank r),
      // slot `split`, as fire-and-forget distributed-shared-memory stores
      const int rpr = kBM / S;
      const uint32_t owner = static_cast<uint32_t>(nl / rpr);
      const uint32_t recv_row =
          smem_u32(base + C::kStageBytes) +
          static_cast<uint32_t>(((split * rpr + nl % rpr) * C::kRedPitch) * 4);
      const uint32_t remote_row = S > 1 ? map_shared_rank(recv_row, owner) : 0u;
      if (S > 1) {
        cluster_wait();
        cluster_waited = true;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < NT; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_d + (static_cast<uint32_t>(quarter * 32) << 16) + c0, r);
        tmem_ld_wait();
        if (S > 1) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_cluster_v4(remote_row + (c0 + 4 * q) * 4,
                                 make_int4(static_cast<int>(r[4 * q]), static_cast<int>(r[4 * q + 1]),
                                           static_cast<int>(r[4 * q + 2]),
                                           static_cast<int>(r[4 * q + 3])));
        } else if (n < N) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int m = m0 + c0 + c;
            if (m < M) {
              const int32_t a = static_cast<int32_t>(r[c]) >> 8;
              if (acc_out) {
                acc_out[static_cast<size_t>(m) * N + n] = a;
              } else {
                const float sc = __ldg(s_x + m) * sw;
                y[static_cast<size_t>(m) * ldy + n] =
                    __float2bfloat16_rn(fmaf(sc, static_cast<float>(a), bn));
              }
            }
          }
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();

  if (S > 1) {
    // ------------------------------------------- cluster split-K reduction
    if (!cluster_waited) cluster_wait();
    cluster_sync();                  // every partial tile has landed
    if (warp >= 2) {
      const int wt = tid - 64;
      const uint32_t rank = cluster_ctarank();
      const int rpr = kBM / S;                     // channel rows reduced by this CTA
      const int32_t* recv = reinterpret_cast<const int32_t*>(base + C::kStageBytes);
      for (int e = wt; e < rpr * NT; e += kWorkers) {
        const int lr = e % rpr;
        const int col = e / rpr;
        int32_t sum = 0;
        for (int src = 0; src < S; ++src) sum += recv[(src * rpr + lr) * C::kRedPitch + col];
        const int nl = rank * rpr + lr;
        const int n = n0 + nl, m = m0 + col;
        if (n < N && m < M) {
          const int32_t a = sum >> 8;
          if (acc_out) {
            acc_out[static_cast<size_t>(m) * N + n] = a;
          } else {
            const float sc = __ldg(s_x + m) * __ldg(s_w + n);
            const float bn = bias != nullptr ? __ldg(bias + n) : 0.f;
            y[static_cast<size_t>(m) * ldy + n] =
                __float2bfloat16_rn(fmaf(sc, static_cast<float>(a), bn));
          }
        }
      }
    }
  }

  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// rows x (K/2) bytes, row pitch K/2; box = 128 bytes x box_rows, 128B swizzle.
bool make_packed_map(CUtensorMap* map, const uint8_t* ptr, int rows, int K, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kRowP), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(ptr), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT>
cudaError_t launch_nt(const GemmArgs& g, int S, cudaStream_t stream) {
  using C = Cfg<NT>;
  if (!C::kCanSplit) S = 1;   // large token tiles supply the parallelism themselves
  CUtensorMap mw, mx;
  if (!make_packed_map(&mw, g.wq, g.N, g.K, kBM) || !make_packed_map(&mx, g.xq, g.M, g.K, NT))
    return cudaErrorInvalidValue;
  auto kern = w4a4_gemm_kernel<NT>;
  static bool attr_set = false;
  cudaError_t e;
  if (!attr_set) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kCanSplit ? C::kSmemBytes + C::kRecvBytes : C::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((g.N + kBM - 1) / kBM, (g.M + NT - 1) / NT, S);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes + (S > 1 ? C::kRecvBytes : 0);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = S;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, mw, mx, g.M, g.N, g.K, g.s_x, g.w_scale, g.bias,
                         static_cast<__nv_bfloat16*>(g.y), g.ldy, g.acc, device_error_word());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int gemm_choose_split(int M, int N, int K) {
  const int nt = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
  if (nt == 256) return 1;
  const int tiles = ((N + kBM - 1) / kBM) * ((M + nt - 1) / nt);
  const int nkt = (K + kKP - 1) / kKP;
  int S = 1;
  while (S < 8 && tiles * S < 148 && 2 * S <= nkt) S *= 2;
  return S;
}

cudaError_t launch_w4a4_gemm(const GemmArgs& g, cudaStream_t stream) {
  int S = g.split_k > 0 ? g.split_k : gemm_choose_split(g.M, g.N, g.K);
  if (g.M <= 16) return launch_nt<16>(g, S, stream);
  if (g.M <= 32) return launch_nt<32>(g, S, stream);
  if (g.M <= 64) return launch_nt<64>(g, S, stream);
  if (g.M <= 128) return launch_nt<128>(g, S, stream);
  return launch_nt<256>(g, S, stream);
}

}  // namespace qvla
