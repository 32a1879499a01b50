// W8A8 GEMM on the sm_100a tensor cores (the W8A8 variant the "FoldQuantVLA"
// page keeps for the attention-output and FFN-down projections):
//
//   acc[m,n] = sum_k q_x[m,k] q_w[n,k]           (int8 x int8 -> int32, exact)
//   y[m,n]   = bf16( fp32(s_x[m] s_w[n]) * acc[m,n] + b[n] )
//
// With one code per byte the tensor core consumes the codes as they are in
// memory: TMA puts 128-byte K slices of the weight rows (128 per tile) and of
// the token rows (NT per tile) into 128-byte-swizzled K-major shared memory,
// which is already the UMMA operand layout, so there is no unpack step.  Warp
// roles: warp 0 issues TMA loads into a ring of kPS stages, one thread of
// warp 1 issues tcgen05.mma kind::i8 (M = 128 weight rows, N = NT tokens,
// K = 32 per instruction) into a tensor-memory accumulator, warps 2-5 read it
// back with tcgen05.ld and apply the epilogue (bf16 tile in shared memory,
// one TMA tensor store; plain stores for a tile cut by N with N % 8 != 0).
// One 128 x NT output tile per CTA, no split-K; one launch takes the tiles of
// up to 16 linears that share the token tile (a CTA finds its linear by the
// prefix sums of their tile counts).
//
// All waits are bounded (2 s) and flag QVLA_DEVERR_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <vector>

#include "qvla_common.cuh"
#include "qvla_internal.h"

namespace qvla {
namespace {

constexpr int kBM = 128;            // weight rows per tile (UMMA M)
constexpr int kKS = 128;            // K (= bytes) per stage
constexpr int kThreads = 192;
constexpr int kWorkers = 128;

template <int NT>
struct W8Cfg {
  static constexpr int kStage = (kBM + NT) * kKS;    // weights, then tokens
  static constexpr int kPS = NT <= 64 ? 6 : (NT == 128 ? 5 : 4);
  static constexpr int kOTile = NT * kBM * 2;        // bf16 [NT][128]
  static constexpr int kSmem = kPS * kStage + 1024;
  static constexpr int kTmemCols = NT < 32 ? 32 : NT;
  static_assert(kOTile <= kPS * kStage, "output tile over the stages");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct W8Problem {
  CUtensorMap tw;                   // int8 weights [N][K], box 128 B x 128 rows
  CUtensorMap tx;                   // int8 codes [M][K], box 128 B x NT rows
  CUtensorMap ty;                   // bf16 output [M][ldy], box 128 channels x NT tokens
  const float* s_x;
  const float* s_w;
  const float* bias;
  __nv_bfloat16* y;
  int32_t* acc;                     // int32 [M][N] output instead of y (tests)
  int M, N, K, ldy, tiles_n;
};
constexpr int kW8MaxBatch = 16;
struct W8Batch {
  int n;
  int tile_start[kW8MaxBatch + 1];  // first CTA of each linear
  W8Problem p[kW8MaxBatch];
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_gemm_kernel(const __grid_constant__ W8Batch batch, unsigned int* err) {
  using C = W8Cfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full[8], empty[8], acc_full;
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(16) float sx_s[NT];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int pi = 0;
  while (pi + 1 < batch.n && static_cast<int>(blockIdx.x) >= batch.tile_start[pi + 1]) ++pi;
  const W8Problem& P = batch.p[pi];
  const int local = static_cast<int>(blockIdx.x) - batch.tile_start[pi];
  const int n0 = (local % P.tiles_n) * kBM;
  const int m0 = (local / P.tiles_n) * NT;
  const int nks = (P.K + kKS - 1) / kKS;
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* const base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);

  if (tid == 0) {
    for (int s = 0; s < C::kPS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    fence_mbar_init();
    tma_prefetch_desc(&P.tw);
    tma_prefetch_desc(&P.tx);
    if (P.acc == nullptr) tma_prefetch_desc(&P.ty);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nks; ++i) {
        const int s = i % C::kPS;
        if (i >= C::kPS && !mbar_wait(&empty[s], ((i / C::kPS) & 1) ^ 1u, err)) break;
        uint8_t* dst = base + s * C::kStage;
        mbar_arrive_expect_tx(&full[s], C::kStage);
        tma_load_2d(dst, &P.tw, &full[s], i * kKS, n0);
        tma_load_2d(dst + kBM * kKS, &P.tx, &full[s], i * kKS, m0);
        ++issued;
      }
      // never leave with copies in flight
      for (int i = issued - C::kPS < 0 ? 0 : issued - C::kPS; i < issued; ++i)
        mbar_wait(&full[i % C::kPS], (i / C::kPS) & 1, err);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, NT);
      for (int i = 0; i < nks; ++i) {
        const int s = i % C::kPS;
        if (!mbar_wait(&full[s], (i / C::kPS) & 1, err)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(base + s * C::kStage);
        const uint32_t b0 = a0 + kBM * kKS;
#pragma unroll
        for (int q = 0; q < kKS / 32; ++q)
          umma_i8(tmem, smem_desc_kmajor_sw128(a0 + 32 * q), smem_desc_kmajor_sw128(b0 + 32 * q),
                  idesc, (i > 0 || q > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(&acc_full);
      mbar_wait(&acc_full, 0, err);      // tensor memory is freed only after this
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int wt = tid - 64;
    const int nl = (warp & 3) * 32 + lane;             // output channel = tensor-memory lane
    const int n = n0 + nl;
    const bool to_y = P.acc == nullptr;
    for (int c = wt; c < NT; c += kWorkers) sx_s[c] = (to_y && m0 + c < P.M) ? P.s_x[m0 + c] : 0.f;
    const float sw = (to_y && n < P.N) ? __ldg(P.s_w + n) : 0.f;
    const float bn = (to_y && n < P.N && P.bias != nullptr) ? __ldg(P.bias + n) : 0.f;
    // one outcome for all workers (they share named barrier 1); also the
    // barrier after which sx_s is complete
    const bool have = named_barrier_all(1, kWorkers, mbar_wait(&acc_full, 0, err));
    __syncwarp();                                      // converged for the warp-wide loads
    tc_fence_after();
    __nv_bfloat16* otile = reinterpret_cast<__nv_bfloat16*>(base);
    if (have) {
#pragma unroll 1
      for (int c0 = 0; c0 < NT; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + c0, r);
        tmem_ld_wait();
        if (!to_y) {
          if (n < P.N)
            for (int c = 0; c < 16; ++c)
              if (m0 + c0 + c < P.M)
                P.acc[static_cast<size_t>(m0 + c0 + c) * P.N + n] = static_cast<int32_t>(r[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c)
            otile[(c0 + c) * kBM + nl] = __float2bfloat16_rn(
                fmaf(sx_s[c0 + c] * sw, static_cast<float>(static_cast<int32_t>(r[c])), bn));
        }
      }
      if (to_y) {
        fence_proxy_async_smem();
        named_barrier(1, kWorkers);
        if (n0 + kBM <= P.N || (P.N & 7) == 0) {
          if (wt == 0) tma_store_2d_and_wait(&P.ty, otile, n0, m0);
        } else {
          // a tile cut by N with N % 8 != 0: plain stores, not a TMA box
          // reaching past N
          for (int e = wt; e < NT * kBM; e += kWorkers) {
            const int c = e / kBM, nx = e % kBM;
            if (n0 + nx < P.N && m0 + c < P.M)
              P.y[static_cast<size_t>(m0 + c) * P.ldy + n0 + nx] = otile[c * kBM + nx];
          }
        }
      }
    }
    tc_fence_before();
  }

  cta_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int NT>
bool fill_w8(W8Problem& P, const GemmArgs& g) {
  std::memset(&P, 0, sizeof(P));
  const uint64_t K = static_cast<uint64_t>(g.K);
  if (!encode_map_2d(&P.tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.wq, K, g.N, K, kKS, kBM,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_2d(&P.tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.xq, K, g.M, K, kKS, NT,
                     CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  if (g.y != nullptr &&
      !encode_map_2d(&P.ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.y, g.N, g.M,
                     static_cast<uint64_t>(g.ldy) * 2, kBM, NT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  P.s_x = g.s_x;
  P.s_w = g.w_scale;
  P.bias = g.bias;
  P.y = static_cast<__nv_bfloat16*>(g.y);
  P.acc = g.y == nullptr ? g.acc : nullptr;
  P.M = g.M;
  P.N = g.N;
  P.K = g.K;
  P.ldy = g.ldy;
  P.tiles_n = (g.N + kBM - 1) / kBM;
  return true;
}

// The linears of one token tile, in launches of at most kW8MaxBatch.
template <int NT>
cudaError_t launch_nt(const std::vector<const GemmArgs*>& gs, cudaStream_t stream) {
  using C = W8Cfg<NT>;
  auto kern = w8a8_gemm_kernel<NT>;
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [&]() {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (e != cudaSuccess) return e;
  for (size_t i0 = 0; i0 < gs.size(); i0 += kW8MaxBatch) {
    const int n = static_cast<int>(std::min<size_t>(kW8MaxBatch, gs.size() - i0));
    W8Batch batch;
    std::memset(&batch, 0, sizeof(batch));
    batch.n = n;
    long long tiles = 0;
    for (int i = 0; i < n; ++i) {
      const GemmArgs& g = *gs[i0 + i];
      if (!fill_w8<NT>(batch.p[i], g)) return cudaErrorInvalidValue;
      batch.tile_start[i] = static_cast<int>(tiles);
      tiles += static_cast<long long>(batch.p[i].tiles_n) * ((g.M + NT - 1) / NT);
    }
    if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    batch.tile_start[n] = static_cast<int>(tiles);
    if (tiles == 0) continue;
    kern<<<static_cast<unsigned>(tiles), kThreads, C::kSmem, stream>>>(batch, device_error_word());
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int w8_token_tile(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

}  // namespace

cudaError_t launch_w8a8_gemm_batch(const GemmArgs* gs, int n, cudaStream_t stream) {
  static const int kTiles[5] = {16, 32, 64, 128, 256};
  for (int t : kTiles) {
    std::vector<const GemmArgs*> grp;
    for (int i = 0; i < n; ++i)
      if (gs[i].M > 0 && w8_token_tile(gs[i].M) == t) grp.push_back(&gs[i]);
    if (grp.empty()) continue;
    cudaError_t e;
    switch (t) {
      case 16: e = launch_nt<16>(grp, stream); break;
      case 32: e = launch_nt<32>(grp, stream); break;
      case 64: e = launch_nt<64>(grp, stream); break;
      case 128: e = launch_nt<128>(grp, stream); break;
      default: e = launch_nt<256>(grp, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_w8a8_gemm(const GemmArgs& g, cudaStream_t stream) {
  return launch_w8a8_gemm_batch(&g, 1, stream);
}

}  // namespace qvla
