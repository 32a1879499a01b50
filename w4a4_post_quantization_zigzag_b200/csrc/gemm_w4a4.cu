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
//   2. unpacks them with four warps into 128-byte-swizzled K-major UMMA
//      operand rows: every code q becomes the int8 value 16*q (its nibble moved into
//      the high half of the byte: `w & 0xF0F0F0F0` for odd codes,
//      `(w << 4) & 0xF0F0F0F0` for even codes).  Even codes of a 32-code
//      group fill the first 16-byte K chunk and odd codes the second; both
//      operands use the same K order, so the dot product is unchanged;
//   3. issues tcgen05.mma kind::i8 (M=128 weight rows, N=NT tokens, K=32)
//      from one thread into an int32 accumulator in tensor memory, which
//      therefore holds 256*acc exactly;
//   4. reads the accumulator back with tcgen05.ld (one output channel per
//      thread, tokens along registers), applies the epilogue into a bf16
//      shared-memory tile and writes it back with one TMA tensor store.
// Weights take the UMMA M slot and tokens the N slot for every M, so the small
// token counts of a DiT action chunk (16-64) still fill a 128-row MMA.
// Small M adds split-K over a thread-block cluster along grid z: every CTA of
// the cluster owns a contiguous run of 256-wide K tiles, and the int32 partial
// tiles are summed through distributed shared memory (exact, no workspace).
//
// All waits are bounded (2 s) and flag QVLA_DEVERR_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <vector>

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
  // split-K receive buffer and the owner's output rows (at most 64 of them,
  // S >= 2), both placed over the stage memory once every CTA of the cluster
  // is done with its stages
  static constexpr int kRecvBytes = kBM * kRedPitch * 4;
  static constexpr int kSmemBytes = kStageBytes + 1024;
  static constexpr bool kCanSplit = kRecvBytes + NT * 64 * 2 <= kStageBytes;
};

struct Barriers {
  uint64_t full_p[4], empty_p[4], full_u[4], empty_u[4], acc_full;
  uint32_t tmem_base;
};

// One linear of a batched launch.  Independent linears (different weights,
// inputs and outputs) share one launch; CTAs are numbered problem by problem.
constexpr int kMaxBatch = 16;
struct GemmProblem {
  CUtensorMap tw;                 // packed weights  [N][K/2]
  CUtensorMap tx;                 // packed codes    [M][K/2]
  CUtensorMap ty;                 // bf16 output [M][ldy], box = (128/S channels) x NT tokens
  const float* s_x;
  const float* s_w;
  const float* bias;
  __nv_bfloat16* y;
  int32_t* acc;
  int M, N, K, ldy;
  int tiles_n;                    // ceil(N / 128)
  int tiles;                      // tiles_n * ceil(M / NT)
  int S;                          // split-K factor: 1 or the launch's cluster size
};
struct GemmBatch {
  int n;
  int tile_start[kMaxBatch + 1];  // prefix sums of tiles_n * tiles_m
  GemmProblem p[kMaxBatch];
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ GemmBatch batch, unsigned int* err) {
  using C = Cfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Barriers bars;
  __shared__ __align__(16) float bars_sx[NT];   // s_x of this token tile

  int pi = 0;
  while (pi + 1 < batch.n && static_cast<int>(blockIdx.x) >= batch.tile_start[pi + 1]) ++pi;
  const GemmProblem& P = batch.p[pi];
  const CUtensorMap* tmap_w = &P.tw;
  const CUtensorMap* tmap_x = &P.tx;
  const int M = P.M, N = P.N, K = P.K, ldy = P.ldy;
  const float* __restrict__ s_x = P.s_x;
  const float* __restrict__ s_w = P.s_w;
  const float* __restrict__ bias = P.bias;
  __nv_bfloat16* __restrict__ y = P.y;
  int32_t* __restrict__ acc_out = P.acc;
  const int local = static_cast<int>(blockIdx.x) - batch.tile_start[pi];
  // A problem with S > 1 spans whole clusters (S consecutive CTAs share a
  // tile, one K range each); a problem with S == 1 is padded to whole
  // clusters, and the padding CTAs leave at once (they take part in no
  // cluster barrier: only split problems use them).
  const int S = P.S;
  if (local >= P.tiles * S) return;
  const int tile = local / S;
  const int split = local % S;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = (tile % P.tiles_n) * kBM;
  const int m0 = (tile / P.tiles_n) * NT;
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
    tma_prefetch_desc(tmap_w);
    tma_prefetch_desc(tmap_x);
  }
  if (warp == 1) {
    __syncwarp();                  // tcgen05 alloc/ld/st/dealloc are warp-wide
    tmem_alloc(&bars.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem_d = bars.tmem_base;
  // split-K: every thread arrives on the cluster barrier once it is done with
  // the stage memory (the producer after its last load has landed, the MMA
  // issuer after its last MMA has completed, the workers after the
  // accumulator is final); partial sums are pushed into the owner's stage
  // memory only after the whole cluster has arrived
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
      for (int i = pre; i < nk; ++i) tma_prefetch_l2_2d(tmap_w, (kt0 + i) * kRowP, n0);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&bars.full_p[i], C::kPStageBytes);
        tma_load_2d(pstage + i * C::kPStageBytes, tmap_w, &bars.full_p[i], (kt0 + i) * kRowP, n0);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        tma_load_2d(pstage + i * C::kPStageBytes + kBM * kRowP, tmap_x, &bars.full_p[i],
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
        tma_load_2d(dst, tmap_w, &bars.full_p[s], xbyte, n0);
        tma_load_2d(dst + kBM * kRowP, tmap_x, &bars.full_p[s], xbyte, m0);
        ++issued;
      }
      // never leave with copies in flight: wait for the last load of each stage
      for (int i = issued - C::kPS < 0 ? 0 : issued - C::kPS; i < issued; ++i)
        mbar_wait(&bars.full_p[i % C::kPS], (i / C::kPS) & 1, err);
    }
    if (S > 1) cluster_arrive_relaxed();
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
          // bytes [32q, 32q+32) of every 128-byte row: the even and the odd
          // codes of packed chunk q of this half stage
          const uint64_t ad = smem_desc_kmajor_sw128(a0 + 32 * q);
          const uint64_t bd = smem_desc_kmajor_sw128(b0 + 32 * q);
          umma_i8(tmem_d, ad, bd, idesc, (j > 0 || q > 0) ? 1u : 0u);
        }
        umma_commit(&bars.empty_u[u]);
      }
      umma_commit(&bars.acc_full);
      mbar_wait(&bars.acc_full, 0, err);   // tensor memory is freed only after this
    }
    if (S > 1) cluster_arrive_relaxed();
  } else {
    // --------------------------------------------------- unpack (4 warps)
    const int wt = tid - 64;   // 0..127
    // epilogue operands, loaded early so their latency hides under the main
    // loop (s_x comes from the previous kernel in the stream)
    pdl_wait();
    float* sx_s = reinterpret_cast<float*>(bars_sx);
    if (acc_out == nullptr)
      for (int c = wt; c < NT; c += kWorkers) sx_s[c] = (m0 + c < M) ? __ldg(s_x + m0 + c) : 0.f;
    const int quarter = warp & 3;
    const int nl = quarter * 32 + lane;          // local output channel (TMEM lane)
    const int n = n0 + nl;
    const float sw = (acc_out == nullptr && n < N) ? __ldg(s_w + n) : 0.f;
    const float bn = (bias != nullptr && n < N) ? __ldg(bias + n) : 0.f;
    constexpr int kItems = (C::kRows * 4 + kWorkers - 1) / kWorkers;
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
        // all packed loads of this half stage first (independent), then the
        // nibble moves and the swizzled 16-byte stores
        uint4 w[kItems];
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
          const int it = wt + k * kWorkers;
          if (it < C::kRows * 4) {
            const int row = ((it >> 5) << 3) + (it & 7);   // A rows, then B rows
            const int cl = (it >> 3) & 3;                  // packed 16-byte chunk of the half
            w[k] = *reinterpret_cast<const uint4*>(ps + row * kRowP +
                                                   (((4 * h + cl) ^ (row & 7)) << 4));
          }
        }
        ok = mbar_wait(&bars.empty_u[u], ((j / C::kUS) & 1) ^ 1u, err);
        if (!ok) break;
        uint8_t* us = ustage + u * C::kUStageBytes;
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
          const int it = wt + k * kWorkers;
          if (it < C::kRows * 4) {
            const int row = ((it >> 5) << 3) + (it & 7);
            const int cl = (it >> 3) & 3;
            uint4 ev, od;
            ev.x = (w[k].x << 4) & 0xF0F0F0F0u;
            ev.y = (w[k].y << 4) & 0xF0F0F0F0u;
            ev.z = (w[k].z << 4) & 0xF0F0F0F0u;
            ev.w = (w[k].w << 4) & 0xF0F0F0F0u;
            od.x = w[k].x & 0xF0F0F0F0u;
            od.y = w[k].y & 0xF0F0F0F0u;
            od.z = w[k].z & 0xF0F0F0F0u;
            od.w = w[k].w & 0xF0F0F0F0u;
            // 128-byte swizzled K-major rows (A rows 0..127, then B rows):
            // chunk 2cl holds the even codes, 2cl+1 the odd codes
            uint8_t* rowp = us + row * kKU;
            *reinterpret_cast<uint4*>(rowp + (((2 * cl) ^ (row & 7)) << 4)) = ev;
            *reinterpret_cast<uint4*>(rowp + (((2 * cl + 1) ^ (row & 7)) << 4)) = od;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars.full_u[u]);
      }
      mbar_arrive(&bars.empty_p[s]);
    }

    // ---------------------------------------------------------- epilogue
    // one outcome per warp, and a converged warp for the warp-wide loads
    const bool have = __all_sync(0xffffffffu, ok && mbar_wait(&bars.acc_full, 0, err));
    tc_fence_after();
    if (S > 1) cluster_arrive_relaxed();
    pdl_launch_dependents();
    if (have) {
      // split-K: this CTA's partial rows go to the receive buffer of the CTA
      // that owns them (rows [r*128/S, (r+1)*128/S) belong to cluster rank r),
      // slot `split`, as fire-and-forget distributed-shared-memory stores
      const int rpr = kBM / S;
      const uint32_t owner = static_cast<uint32_t>(nl / rpr);
      const uint32_t recv_row =
          smem_u32(base) + static_cast<uint32_t>(((split * rpr + nl % rpr) * C::kRedPitch) * 4);
      const uint32_t remote_row = S > 1 ? map_shared_rank(recv_row, owner) : 0u;
      if (S > 1) {
        cluster_wait();
        cluster_waited = true;
      }
      // bf16 output tile [NT tokens][128 channels] in the (now idle) stage
      // memory, written back by one TMA tensor store
      __nv_bfloat16* otile = reinterpret_cast<__nv_bfloat16*>(base);
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
        } else if (acc_out) {
          if (n < N) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int m = m0 + c0 + c;
              if (m < M) acc_out[static_cast<size_t>(m) * N + n] = static_cast<int32_t>(r[c]) >> 8;
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float sc = sx_s[c0 + c] * sw;
            const int32_t a = static_cast<int32_t>(r[c]) >> 8;
            otile[(c0 + c) * kBM + nl] = __float2bfloat16_rn(fmaf(sc, static_cast<float>(a), bn));
          }
        }
      }
      if (S == 1 && acc_out == nullptr) {
        fence_proxy_async_smem();
        named_barrier(1, kWorkers);
        if (n0 + kBM <= N || (N & 7) == 0) {
          if (wt == 0) tma_store_2d_and_wait(&P.ty, otile, n0, m0);
        } else {
          // a tile cut by N with N % 8 != 0: plain stores, not a TMA box
          // reaching past N
          for (int e = wt; e < NT * kBM; e += kWorkers) {
            const int c = e / kBM, nx = e % kBM;
            if (n0 + nx < N && m0 + c < M)
              y[static_cast<size_t>(m0 + c) * ldy + n0 + nx] = otile[c * kBM + nx];
          }
        }
      }
    }
    tc_fence_before();
  }

  cta_sync();

  if (S > 1) {
    // ------------------------------------------- cluster split-K reduction
    if (!cluster_waited) cluster_wait();
    cluster_sync();                  // every partial tile has landed
    if (warp >= 2) {
      const int wt = tid - 64;
      const uint32_t rank = cluster_ctarank();
      const int rpr = kBM / S;                     // channel rows reduced by this CTA
      const int32_t* recv = reinterpret_cast<const int32_t*>(base);
      // output tile [NT tokens][rpr channels] for one TMA store of this CTA's
      // rows, after the receive buffer
      __nv_bfloat16* otile = reinterpret_cast<__nv_bfloat16*>(base + C::kRecvBytes);
      for (int e = wt; e < rpr * NT; e += kWorkers) {
        const int lr = e % rpr;
        const int col = e / rpr;
        int32_t sum = 0;
        for (int src = 0; src < S; ++src) sum += recv[(src * rpr + lr) * C::kRedPitch + col];
        const int nl = rank * rpr + lr;
        const int n = n0 + nl, m = m0 + col;
        const int32_t a = sum >> 8;
        if (acc_out) {
          if (n < N && m < M) acc_out[static_cast<size_t>(m) * N + n] = a;
        } else {
          const float sc = n < N ? bars_sx[col] * __ldg(s_w + n) : 0.f;
          const float bn = (bias != nullptr && n < N) ? __ldg(bias + n) : 0.f;
          otile[col * rpr + lr] = __float2bfloat16_rn(fmaf(sc, static_cast<float>(a), bn));
        }
      }
      if (acc_out == nullptr) {
        fence_proxy_async_smem();
        named_barrier(1, kWorkers);
        const int nr = n0 + static_cast<int>(rank) * rpr;
        if (nr + rpr <= N || (N & 7) == 0) {
          if (wt == 0) tma_store_2d_and_wait(&P.ty, otile, nr, m0);
        } else {
          for (int e = wt; e < NT * rpr; e += kWorkers) {
            const int c = e / rpr, nx = e % rpr;
            if (nr + nx < N && m0 + c < M)
              y[static_cast<size_t>(m0 + c) * ldy + nr + nx] = otile[c * rpr + nx];
          }
        }
      }
    }
  }

  if (warp == 1) {
    __syncwarp();                  // lane 0 comes from the MMA loop
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
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
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

// bf16 [M][ldy] output; box = box_n channels x box_m tokens, no swizzle.
bool make_output_map(CUtensorMap* map, void* ptr, int M, int N, int ldy, int box_n, int box_m) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldy) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_n), static_cast<cuuint32_t>(box_m)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT>
cudaError_t launch_group(const GemmArgs* const* gs, const int* splits, int n, int C,
                         cudaStream_t stream) {
  using C_ = Cfg<NT>;
  GemmBatch batch;
  std::memset(&batch, 0, sizeof(batch));
  batch.n = n;
  int ctas = 0;
  for (int i = 0; i < n; ++i) {
    const GemmArgs& g = *gs[i];
    GemmProblem& P = batch.p[i];
    const int S = splits[i];
    if (!make_packed_map(&P.tw, g.wq, g.N, g.K, kBM) || !make_packed_map(&P.tx, g.xq, g.M, g.K, NT))
      return cudaErrorInvalidValue;
    if (g.y != nullptr && !make_output_map(&P.ty, g.y, g.M, g.N, g.ldy, kBM / S, NT))
      return cudaErrorInvalidValue;
    P.s_x = g.s_x;
    P.s_w = g.w_scale;
    P.bias = g.bias;
    P.y = static_cast<__nv_bfloat16*>(g.y);
    P.acc = g.acc;
    P.M = g.M;
    P.N = g.N;
    P.K = g.K;
    P.ldy = g.ldy;
    P.tiles_n = (g.N + kBM - 1) / kBM;
    P.tiles = P.tiles_n * ((g.M + NT - 1) / NT);
    P.S = S;
    batch.tile_start[i] = ctas;
    ctas += (P.tiles * S + C - 1) / C * C;     // whole clusters
  }
  batch.tile_start[n] = ctas;
  auto kern = w4a4_gemm_kernel<NT>;
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [&]() {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C_::kSmemBytes);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return r;
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C_::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (C > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = C;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, batch, device_error_word());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

int token_tile(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

// Split-K factors of a launch (1 or the launch's cluster size C per problem).
// Requested: the same factor everywhere.  Automatic: one factor for all,
// raised while the launch has fewer CTAs than SMs.
template <int NT>
int choose_splits(const GemmArgs* const* gs, int n, int split_k, int* splits) {
  if (!Cfg<NT>::kCanSplit) {
    for (int i = 0; i < n; ++i) splits[i] = 1;
    return 1;
  }
  if (split_k > 0) {
    for (int i = 0; i < n; ++i) splits[i] = split_k;
    return split_k;
  }
  int min_nkt = 1 << 30, max_nkt = 0;
  for (int i = 0; i < n; ++i) {
    const int nkt = (gs[i]->K + kKP - 1) / kKP;
    min_nkt = std::min(min_nkt, nkt);
    max_nkt = std::max(max_nkt, nkt);
  }
  for (int i = 0; i < n; ++i) splits[i] = 1;
  if (NT <= 64 && max_nkt > 2 * min_nkt) {
    // Weight-streaming launches (few tokens): linears more than twice as deep
    // in K as the shallowest of the launch are split over a cluster of C
    // CTAs, so that no CTA walks more than about twice the K tiles of the
    // shallowest; the others stay whole.  (The split costs no extra shared
    // memory: partial sums land in the stage memory of the owner once the
    // cluster is done with its stages.)  With many tokens the launch already
    // has several waves of CTAs and splitting measured slower.
    int C = 1;
    while (C < 8 && max_nkt > 2 * min_nkt * C) C *= 2;
    for (int i = 0; i < n; ++i) {
      const int nkt = (gs[i]->K + kKP - 1) / kKP;
      if (nkt > 2 * min_nkt && C <= nkt) splits[i] = C;
    }
    return C;
  }
  // similar depths: one factor for all, raised while the launch has fewer
  // CTAs than SMs
  int C = 1;
  auto total = [&]() {
    int t = 0;
    for (int i = 0; i < n; ++i)
      t += ((gs[i]->N + kBM - 1) / kBM) * ((gs[i]->M + NT - 1) / NT) * splits[i];
    return t;
  };
  while (C < 8 && total() < 148 && 2 * C <= min_nkt) {
    C *= 2;
    for (int i = 0; i < n; ++i) splits[i] = C;
  }
  return C;
}

template <int NT>
cudaError_t launch_nt_batches(const GemmArgs* const* gs, int n, int split_k, cudaStream_t stream) {
  // (Giving the deepest linears of a batch a launch of their own, with their
  // own split-K factor, balances the K walk per CTA but measured slower on
  // the DiT shapes: each extra launch costs more than the imbalance.)
  for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
    const int m = std::min(kMaxBatch, n - i0);
    int splits[kMaxBatch];
    const int C = choose_splits<NT>(gs + i0, m, split_k, splits);
    // CTAs are dispatched in index order: the split (deepest) linears first,
    // so that a partial second wave holds only short CTAs
    const GemmArgs* order[kMaxBatch];
    int osplit[kMaxBatch];
    int k = 0;
    for (int pass = 0; pass < 2; ++pass)
      for (int i = 0; i < m; ++i)
        if ((splits[i] > 1) == (pass == 0)) {
          order[k] = gs[i0 + i];
          osplit[k++] = splits[i];
        }
    cudaError_t e = launch_group<NT>(order, osplit, m, C, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

bool encode_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t inner,
                   uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemm_choose_split(int M, int N, int K) {
  const int nt = token_tile(M);
  if (nt == 256) return 1;
  const int tiles = ((N + kBM - 1) / kBM) * ((M + nt - 1) / nt);
  const int nkt = (K + kKP - 1) / kKP;
  int S = 1;
  while (S < 8 && tiles * S < 148 && 2 * S <= nkt) S *= 2;
  return S;
}

cudaError_t launch_w4a4_gemm_batch(const GemmArgs* gs, int n, int split_k, cudaStream_t stream) {
  // group by token tile (a template parameter of the kernel)
  static const int kTiles[5] = {16, 32, 64, 128, 256};
  for (int t : kTiles) {
    std::vector<const GemmArgs*> grp;
    for (int i = 0; i < n; ++i)
      if (gs[i].M > 0 && token_tile(gs[i].M) == t) grp.push_back(&gs[i]);
    if (grp.empty()) continue;
    cudaError_t e;
    switch (t) {
      case 16: e = launch_nt_batches<16>(grp.data(), static_cast<int>(grp.size()), split_k, stream); break;
      case 32: e = launch_nt_batches<32>(grp.data(), static_cast<int>(grp.size()), split_k, stream); break;
      case 64: e = launch_nt_batches<64>(grp.data(), static_cast<int>(grp.size()), split_k, stream); break;
      case 128: e = launch_nt_batches<128>(grp.data(), static_cast<int>(grp.size()), split_k, stream); break;
      default: e = launch_nt_batches<256>(grp.data(), static_cast<int>(grp.size()), split_k, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_w4a4_gemm(const GemmArgs& g, cudaStream_t stream) {
  return launch_w4a4_gemm_batch(&g, 1, g.split_k, stream);
}

}  // namespace qvla
