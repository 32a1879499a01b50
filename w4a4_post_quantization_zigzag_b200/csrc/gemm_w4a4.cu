// W4A4 GEMM on the sm_100a tensor cores with a fused dequantisation epilogue.
//
//   acc[m,n] = sum_k q_x[m,k] q_w[n,k]                      (exact)
//   y[m,n]   = bf16( fp32(s_x[m] s_w[n]) * acc[m,n] + b[n] )
//
// ("Omega-QVLA: Nen VLA W4A4 tren Edge", section "Vi sao W4A4 kho hon
// W4A16?": weights and activations both 4-bit so the product runs on integer
// tensor cores; "FoldQuantVLA": native integer W4A4 execution.)
//
// sm_100a has no 4-bit integer MMA.  Every code q runs through
// tcgen05.mma kind::i8 as the int8 value 16*q (its nibble moved into the high
// half of the byte: `w & 0xF0F0F0F0` takes the odd codes of a packed word,
// `(w << 4) & 0xF0F0F0F0` the even ones), so the int32 accumulator holds
// 256*acc exactly and the epilogue shifts it back.  Inside every group of 32
// codes both operands carry the even codes first, then the odd ones; the dot
// product is unchanged.
//
// One persistent CTA per SM, warp-specialised (320 threads):
//   warp 0      TMA producer: per pipeline stage (256 of K) a 128-row box of
//               packed weights and the NT-token activation box(es) go into a
//               ring of shared-memory stages;
//   warp 1      MMA issuer: tcgen05.mma with A (weights) read from tensor
//               memory and B (activations) from shared memory, eight K = 32
//               MMAs and one commit per stage; int32 accumulators in tensor
//               memory, two buffers when they fit;
//   warps 2-5   unpack: each thread owns one weight row (one tensor-memory
//               lane), reads the row's 128 packed bytes of the stage and
//               stores its 256 int8 values into the stage's tensor-memory A
//               slot (tcgen05.st), so the weights never make a second trip
//               through shared memory; with nibble-packed activations these
//               warps also unpack the B tile into 128-byte-swizzled shared
//               memory;
//   warps 6-9   epilogue: tcgen05.ld of the accumulator (one output channel per
//               thread), dequantise, add the bias, round to bf16, stage
//               32-token chunks in shared memory, TMA tensor stores.
// Shared-memory stage s and tensor-memory A slot s form one ring: the unpack
// warps' arrival says both that the stage's bytes were read and that its A is
// ready, and one MMA commit frees both.
// The activation operand is either the int8 image of the codes written by the
// rotate-quantise step (16*q, the same order inside each 32-code group; a TMA
// box lands directly in the MMA layout) or the nibble-packed codes.
// Tiles (128 weight rows x NT tokens x all of K) are dealt to the CTAs on the
// host, longest first to the least-loaded CTA, and travel in the kernel
// parameters; a CTA walks its list with one continuous pipeline, so the next
// tile's loads and unpacking overlap the current tile's MMAs and the previous
// tile's epilogue.
//
// All waits are bounded (2 s) and flag QVLA_DEVERR_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <queue>
#include <vector>

#include "qvla_common.cuh"
#include "qvla_internal.h"

namespace qvla {
namespace {

constexpr int kBM = 128;                  // weight rows per tile (UMMA M, tensor-memory lanes)
constexpr int kKS = 256;                  // K per pipeline stage
constexpr int kAPack = kKS / 2;           // packed weight bytes per row per stage (one 128B-swizzled box)
constexpr int kACols = kKS / 4;           // tensor-memory columns of one unpacked A stage
constexpr int kBaseThreads = 320;
constexpr int kOutSlots = 4;              // output staging ring (32-token chunks)
constexpr int kTmemCols = 512;
constexpr int kMaxBatch = 16;
constexpr int kMaxTiles = 2048;
constexpr int kMaxCtas = 160;
constexpr uint32_t kFull = 0xffffffffu;

template <int NT, bool kImage>
struct Cfg {
  static constexpr int kAcc = NT >= 256 ? 1 : 2;                  // accumulator buffers
  static constexpr int kAccCols = NT < 32 ? 32 : NT;
  // MMA issuers: with small token tiles a second thread issues every other
  // stage of a tile into its own accumulator (the epilogue adds the two), so
  // that the tensor pipe runs one issuer's MMAs while the other waits
  static constexpr int kIss = NT <= 64 ? 2 : 1;
  static constexpr int kThreads = kBaseThreads + 32 * (kIss - 1);  // warp 10: second issuer
  static constexpr int kACol0 = kAcc * kIss * kAccCols;          // first A-stage column
  static constexpr int kABytes = kBM * kAPack;                   // packed weight box
  // activations: the image as two 128-byte boxes (K halves) of NT rows, or
  // one 128-byte box of packed codes plus their unpacked two halves
  static constexpr int kBBytes = kImage ? 2 * NT * 128 : NT * 128;
  static constexpr int kUBytes = kImage ? 0 : 2 * NT * 128;
  static constexpr int kStage = kABytes + kBBytes + kUBytes;
  static constexpr int kCh = NT < 32 ? NT : 32;                  // tokens per output chunk
  static constexpr int kOutBytes = kOutSlots * kCh * kBM * 2;
  // small token tiles may split the K of a long tile over the two CTAs of a
  // cluster: the second CTA's int32 partial lands in the first one's
  // receive buffer, [token / 4][weight row][4 tokens]
  static constexpr bool kSplit = NT <= 64;
  static constexpr int kRecvBytes = kSplit ? kBM * NT * 4 : 0;
  static constexpr int kBudget = 226 * 1024;                     // dynamic shared memory
  static constexpr int kRing = (kBudget - 1024 - kOutBytes - kRecvBytes) / kStage;
  static constexpr int kTmemStages = (kTmemCols - kACol0) / kACols;
  static constexpr int kS0 = kRing < kTmemStages ? kRing : kTmemStages;
  // one ring: smem stage s and tensor-memory A stage s go together
  static constexpr int kS = kS0 > 8 ? 8 : kS0;
  // at least 116 KB, so that two CTAs never share an SM (each takes all of
  // tensor memory)
  static constexpr int kNeed = kS * kStage + kOutBytes + kRecvBytes + 1024;
  static constexpr int kSmem = kNeed < 116 * 1024 ? 116 * 1024 : kNeed;
  static_assert(kACol0 + kS * kACols <= kTmemCols, "tensor memory");
  static_assert(kStage % 1024 == 0 && kABytes % 1024 == 0 && kBBytes % 1024 == 0, "alignment");
  static_assert(kS >= 2, "pipeline depth");
  static_assert(kNeed <= kBudget, "shared memory");
};

struct Barriers {
  uint64_t full[8];                        // TMA: packed weights and activations landed
  uint64_t unp_done[8];                    // the four unpack warps are done with the stage
  uint64_t mma_done[8];                    // the MMAs reading the stage have completed
  uint64_t acc_full[2], acc_empty[2];      // accumulators
  uint64_t drain;
  uint64_t recv_full;                      // the cluster partner's partial has landed
  uint32_t tmem;
};

// One linear of a launch.  Its tiles are numbered n-tile fastest (tiles that
// share an activation box are neighbours), from tile_base on.
struct Problem {
  CUtensorMap tw;                 // packed weights [N][K/2]: box 128 B x 128 rows, 128B swizzle
  CUtensorMap tx;                 // activations: int8 image [M][K] or packed [M][K/2], box
                                  // 128 B x NT rows, 128B swizzle
  CUtensorMap ty;                 // bf16 output [M][ldy]: box 128 channels x kCh tokens
  const float* s_x;
  const float* s_w;
  const float* bias;
  __nv_bfloat16* y;
  int32_t* acc;                   // int32 [M][N] accumulators instead of y (or null)
  int M, N, K, ldy;
  int tiles_n;                    // ceil(N / 128)
  int nks;                        // K stages: ceil(K / 256)
  int tile_base;                  // first tile of this problem in the launch
};
struct Batch {
  int n;
  int split;                      // launched in clusters of two CTAs
  int tile_start[kMaxBatch + 1];  // launch tile ids of each problem
  uint16_t cta_begin[kMaxCtas + 1];
  // the tiles, CTA by CTA (a split tile twice), each packed as
  // problem | n-tile << 4 | m-tile << 19
  uint32_t order[kMaxTiles + kMaxCtas];
  // with `split`, the role of each CTA's first tile: 0 the whole tile, 1 its
  // first K half and the epilogue (cluster rank 0), 2 its second K half,
  // sent to rank 0 (cluster rank 1)
  int8_t role[kMaxCtas];
  Problem p[kMaxBatch];
};

struct Tile {
  int p, n0, m0;
};

template <int NT>
QVLA_DEVICE Tile decode(uint32_t w) {
  return Tile{static_cast<int>(w & 15u), static_cast<int>((w >> 4) & 0x7FFFu) * kBM,
              static_cast<int>(w >> 19) * NT};
}
constexpr int kListCache = 64;            // list entries a CTA keeps in shared memory

// Wait until at most N bulk groups of this thread still read shared memory.
template <int N>
QVLA_DEVICE void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int NT>
QVLA_DEVICE void tmem_ld_chunk(uint32_t taddr, uint32_t (&r)[NT < 32 ? NT : 32]) {
  if constexpr (NT < 32) {
    tmem_ld16(taddr, r);
  } else {
    tmem_ld32(taddr, r);
  }
}

// 16 packed bytes (32 codes) -> 8 words of 16*q int8: the even codes of the
// four words, then the odd codes.
QVLA_DEVICE void unpack32(const uint4 v, uint32_t* o) {
  o[0] = (v.x << 4) & 0xF0F0F0F0u;
  o[1] = (v.y << 4) & 0xF0F0F0F0u;
  o[2] = (v.z << 4) & 0xF0F0F0F0u;
  o[3] = (v.w << 4) & 0xF0F0F0F0u;
  o[4] = v.x & 0xF0F0F0F0u;
  o[5] = v.y & 0xF0F0F0F0u;
  o[6] = v.z & 0xF0F0F0F0u;
  o[7] = v.w & 0xF0F0F0F0u;
}

template <int NT, bool kImage>
__global__ void __launch_bounds__(Cfg<NT, kImage>::kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ Batch batch, unsigned int* err) {
  using C = Cfg<NT, kImage>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Barriers bars;
  __shared__ __align__(16) float sx_s[NT];       // s_x of the epilogue's current tile
  // the head of the CTA's tile list and the problems' stage counts, read from
  // the kernel parameters once by one warp (every role walks the list)
  __shared__ uint32_t list_s[kListCache];
  __shared__ uint8_t nks_s[kMaxBatch];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t_begin = batch.cta_begin[blockIdx.x];
  const int t_end = batch.cta_begin[blockIdx.x + 1];
  auto tile_at = [&](int i) -> Tile {
    const int j = i - t_begin;
    return decode<NT>(j < kListCache ? list_s[j] : batch.order[i]);
  };
  // K stages [k0, k1) of the CTA's i-th tile: all of them, or one half when
  // the tile is split over the cluster pair
  const int role = (C::kSplit && batch.split) ? batch.role[blockIdx.x] : 0;
  auto krange = [&](int i, int nks, int& k0, int& k1) {
    k0 = 0;
    k1 = nks;
    if (role != 0 && i == t_begin) {
      if (role == 1) k1 = nks / 2;
      else k0 = nks / 2;
    }
  };

  // 1024-byte aligned stage memory (128B-swizzled TMA destinations)
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* const base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* const stages = base;
  __nv_bfloat16* const outs = reinterpret_cast<__nv_bfloat16*>(base + C::kS * C::kStage);
  uint8_t* const recv = base + C::kS * C::kStage + C::kOutBytes;

  constexpr uint32_t kTx = C::kABytes + C::kBBytes;
  int pre = 0;                                   // stages the producer issued during setup
  if (tid == 0) {
    for (int s = 0; s < C::kS; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.unp_done[s], 4);
      mbar_init(&bars.mma_done[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], C::kIss);
      mbar_init(&bars.acc_empty[b], 4);
    }
    mbar_init(&bars.drain, C::kIss);
    mbar_init(&bars.recv_full, 1);
    fence_mbar_init();
    for (int p = 0; p < batch.n; ++p) {
      tma_prefetch_desc(&batch.p[p].tw);
      tma_prefetch_desc(&batch.p[p].tx);
    }
    // The producer's ramp, while the other warps set up: the first ring's
    // worth of weight boxes (they do not depend on the previous kernel in the
    // stream), then, once that kernel is done (programmatic dependent
    // launch), the same stages' activation boxes.
    for (int pass = 0; pass < 2; ++pass) {
      int i = t_begin, ks = -1, n = 0;
      while (n < C::kS && i < t_end) {
        const Tile tr = decode<NT>(batch.order[i]);
        const Problem& P = batch.p[tr.p];
        int k0, k1;
        krange(i, P.nks, k0, k1);
        if (ks < 0) ks = k0;
        uint8_t* st = stages + n * C::kStage;
        if (pass == 0) {
          mbar_arrive_expect_tx(&bars.full[n], kTx);
          tma_load_2d(st, &P.tw, &bars.full[n], ks * kAPack, tr.n0);
        } else if constexpr (kImage) {
          tma_load_2d(st + C::kABytes, &P.tx, &bars.full[n], ks * kKS, tr.m0);
          tma_load_2d(st + C::kABytes + NT * 128, &P.tx, &bars.full[n], ks * kKS + 128, tr.m0);
        } else {
          tma_load_2d(st + C::kABytes, &P.tx, &bars.full[n], ks * kAPack, tr.m0);
        }
        ++n;
        if (++ks == k1) {
          ks = -1;
          ++i;
        }
      }
      pre = n;
      if (pass == 0) pdl_wait();
    }
  }
  if (warp == 1) {
    __syncwarp();                  // tcgen05 alloc/ld/st/dealloc are warp-wide
    tmem_alloc(&bars.tmem, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) {
    for (int j = lane; j < kListCache && t_begin + j < t_end; j += 32) list_s[j] = batch.order[t_begin + j];
    if (lane < batch.n) nks_s[lane] = static_cast<uint8_t>(batch.p[lane].nks);
  }
  tc_fence_before();
  cta_sync();
  // cluster barrier phase 1 ("barriers initialised"): every thread arrives
  // now; a thread waits for it only before its first access to the
  // partner's shared memory, or at the end
  if (batch.split) cluster_arrive_release();
  bool cluster_waited = false;
  tc_fence_after();
  const uint32_t tmem = bars.tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // past the stages issued during setup
      bool ok = true;
      int g = 0;
      for (int i = t_begin; i < t_end && ok; ++i) {
        const Tile tr = tile_at(i);
        const Problem& P = batch.p[tr.p];
        int k0, k1;
        krange(i, nks_s[tr.p], k0, k1);
        // the tile's weight boxes past the ring depth go to L2 now, so HBM
        // streaming is not limited by the ring
        for (int ks = k0 + C::kS; ks < k1; ++ks) tma_prefetch_l2_2d(&P.tw, ks * kAPack, tr.n0);
        for (int ks = k0; ks < k1; ++ks, ++g) {
          const int s = g % C::kS;
          uint8_t* st = stages + s * C::kStage;
          if (g >= pre) {
            if (g >= C::kS) {
              // the unpack warps have read the stage and the MMAs are done with it
              const uint32_t ph = ((g / C::kS) - 1) & 1;
              ok = mbar_wait(&bars.unp_done[s], ph, err) && mbar_wait(&bars.mma_done[s], ph, err);
              if (!ok) break;
            }
            mbar_arrive_expect_tx(&bars.full[s], kTx);
            tma_load_2d(st, &P.tw, &bars.full[s], ks * kAPack, tr.n0);
            if constexpr (kImage) {
              tma_load_2d(st + C::kABytes, &P.tx, &bars.full[s], ks * kKS, tr.m0);
              tma_load_2d(st + C::kABytes + NT * 128, &P.tx, &bars.full[s], ks * kKS + 128, tr.m0);
            } else {
              tma_load_2d(st + C::kABytes, &P.tx, &bars.full[s], ks * kAPack, tr.m0);
            }
          }
        }
      }
      // never leave with copies in flight: the last load of every stage has landed
      for (int j = g - C::kS < 0 ? 0 : g - C::kS; j < g; ++j)
        mbar_wait(&bars.full[j % C::kS], (j / C::kS) & 1, err);
    }
  } else if (warp == 1 || (C::kIss == 2 && warp == kBaseThreads / 32)) {
    // ------------------------------------------------------------- MMA issuers
    // issuer j takes the stages ks of each tile with (ks - k0) % kIss == j,
    // into accumulator column block (b * kIss + j)
    if (lane == 0) {
      const int j = warp == 1 ? 0 : 1;
      constexpr uint32_t idesc = idesc_i8(kBM, NT);
      bool ok = true;
      int g = 0, tc = 0;
      for (int i = t_begin; i < t_end && ok; ++i, ++tc) {
        const Tile tr = tile_at(i);
        int k0, k1;
        krange(i, nks_s[tr.p], k0, k1);
        const int b = tc % C::kAcc, use = tc / C::kAcc;
        if (use >= 1) {
          ok = mbar_wait(&bars.acc_empty[b], (use - 1) & 1, err);
          if (!ok) break;
        }
        const uint32_t d = tmem + static_cast<uint32_t>((b * C::kIss + j) * C::kAccCols);
        for (int ks = k0; ks < k1; ++ks, ++g) {
          if ((ks - k0) % C::kIss != j) continue;         // the other issuer's stage
          const int s = g % C::kS;
          // the stage's A is in tensor memory (and, when the unpack warps got
          // the stage, its TMA bytes, activations included, had landed)
          ok = mbar_wait(&bars.unp_done[s], (g / C::kS) & 1, err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bs =
              smem_u32(stages + s * C::kStage + C::kABytes + (kImage ? 0 : C::kBBytes));
          const uint32_t at = tmem + static_cast<uint32_t>(C::kACol0 + s * kACols);
#pragma unroll
          for (int kk = 0; kk < kKS / 32; ++kk) {
            // 32 codes of K: A columns [8kk, 8kk+8) of the stage; B half kk/4,
            // bytes [32(kk%4), +32) of each 128-byte row
            const uint64_t bd = smem_desc_kmajor_sw128(bs + (kk >> 2) * (NT * 128) + 32 * (kk & 3));
            umma_i8_tmem_a(d, at + 8 * kk, bd, idesc, (ks >= k0 + C::kIss || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars.mma_done[s]);
        }
        if (!ok) break;
        // (an issuer without a stage in this tile still arrives: its
        // accumulator is then not read)
        umma_commit(&bars.acc_full[b]);
      }
      umma_commit(&bars.drain);
      mbar_wait(&bars.drain, 0, err);   // tensor memory is freed only after this
    }
  } else if (warp < 6) {
    // ------------------------------------------------------- unpack (4 warps)
    const int q4 = warp & 3;                       // tensor-memory lane quarter
    const int row = q4 * 32 + lane;                // weight row of the tile
    const int wt = tid - 64;                       // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    constexpr int kBItems = (NT * 8 + 127) / 128;  // packed activation chunks per thread
    bool ok = true;
    int g = 0;
    for (int i = t_begin; i < t_end && ok; ++i) {
      int k0, k1;
      krange(i, nks_s[tile_at(i).p], k0, k1);
      for (int ks = k0; ks < k1; ++ks, ++g) {
        const int s = g % C::kS;
        // warp-uniform outcome: the tensor-memory stores below are warp-wide
        ok = __all_sync(kFull, mbar_wait(&bars.full[s], (g / C::kS) & 1, err));
        if (!ok) break;
        const uint32_t st = smem_u32(stages + s * C::kStage);
        // the row's 128 packed bytes; 128-byte swizzle: 16-byte chunk c of row
        // r sits at chunk c ^ (r & 7)
        uint4 w[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) w[c] = lds128(st + row * kAPack + ((c ^ (row & 7)) << 4));
        // the previous use of this stage (tensor-memory A, unpacked activations)
        // is over once its MMAs have completed
        if (g >= C::kS) {
          ok = __all_sync(kFull, mbar_wait(&bars.mma_done[s], ((g / C::kS) - 1) & 1, err));
          if (!ok) break;
        }
        tc_fence_after();
        if constexpr (!kImage) {
          // activation chunk e: code row br = e % NT, 32-code group c = e / NT
          // (consecutive threads take consecutive rows: conflict-free); group
          // c goes to K half c / 4 as 16-byte chunks 2(c%4) (even codes) and
          // 2(c%4)+1 (odd codes) of a 128-byte swizzled row
          const uint32_t bp = st + C::kABytes, bu = st + C::kABytes + C::kBBytes;
#pragma unroll
          for (int k = 0; k < kBItems; ++k) {
            const int e = wt + k * 128;
            if (e < NT * 8) {
              const int br = e % NT, c = e / NT;
              const uint4 v = lds128(bp + br * 128 + ((c ^ (br & 7)) << 4));
              uint32_t o[8];
              unpack32(v, o);
              const uint32_t rowp = bu + (c >> 2) * (NT * 128) + br * 128;
              const int cl = c & 3;
              sts128(rowp + (((2 * cl) ^ (br & 7)) << 4), make_uint4(o[0], o[1], o[2], o[3]));
              sts128(rowp + (((2 * cl + 1) ^ (br & 7)) << 4), make_uint4(o[4], o[5], o[6], o[7]));
            }
          }
        }
        // 64 columns: packed chunk c -> columns [8c, 8c+8)
        const uint32_t ta = tmem + lane_base + static_cast<uint32_t>(C::kACol0 + s * kACols);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t av[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) unpack32(w[4 * h + c], av + 8 * c);
          tmem_st32(ta + 32 * h, av);
        }
        tmem_st_wait();
        if constexpr (!kImage) fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.unp_done[s]);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;                // output channel of the tile
    const int et = tid - 192;                      // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    pdl_wait();                                    // s_x comes from the previous kernel
    bool ok = true;
    int tc = 0, chunk = 0;
    for (int i = t_begin; i < t_end && ok; ++i, ++tc) {
      const Tile tr = tile_at(i);
      const Problem& P = batch.p[tr.p];
      const int b = tc % C::kAcc, use = tc / C::kAcc;
      // the tile's token scales, output-channel scale and bias, loaded while
      // its MMAs run (the previous tile's readers of sx_s all passed the
      // barrier that closed its last chunk)
      const int n = tr.n0 + row;
      const bool nv = n < P.N;
      const float sw = (P.acc == nullptr && nv) ? __ldg(P.s_w + n) : 0.f;
      const float bn = (P.bias != nullptr && nv) ? __ldg(P.bias + n) : 0.f;
      if (P.acc == nullptr)
        for (int j = et; j < NT; j += 128) sx_s[j] = tr.m0 + j < P.M ? __ldg(P.s_x + tr.m0 + j) : 0.f;
      // one outcome for all four epilogue warps (they share named barriers);
      // also publishes sx_s
      ok = named_barrier_all(2, 128, mbar_wait(&bars.acc_full[b], use & 1, err));
      if (!ok) break;
      tc_fence_after();
      const bool tma = tr.n0 + kBM <= P.N || (P.N & 7) == 0;
      const uint32_t tacc = tmem + lane_base + static_cast<uint32_t>(b * C::kIss * C::kAccCols);
      const bool first = i == t_begin;
      // the second issuer's accumulator holds stages when the tile has two or more
      int k0, k1;
      krange(i, nks_s[tr.p], k0, k1);
      const bool two = C::kIss == 2 && k1 - k0 >= 2;
      auto load_acc = [&](int c0, uint32_t (&r)[C::kCh]) {
        tmem_ld_chunk<NT>(tacc + c0, r);
        tmem_ld_wait();
        if (two) {
          uint32_t r2[C::kCh];
          tmem_ld_chunk<NT>(tacc + C::kAccCols + c0, r2);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < C::kCh; ++q) r[q] += r2[q];
        }
      };
      if (role == 2 && first) {
        // second K half of a split tile: the int32 partial goes to the
        // receive buffer of cluster rank 0; once all four warps have stored
        // theirs (the barrier orders them before the release), one thread
        // arrives on rank 0's barrier, releasing at cluster scope
        const uint32_t rv = map_shared_rank(smem_u32(recv), 0u);
        cluster_wait();
        cluster_waited = true;
#pragma unroll 1
        for (int c0 = 0; c0 < NT; c0 += C::kCh) {
          uint32_t r[C::kCh];
          load_acc(c0, r);
#pragma unroll
          for (int j = 0; j < C::kCh; j += 4)
            st_shared_cluster_v4(rv + static_cast<uint32_t>((((c0 + j) >> 2) * kBM + row) * 16),
                                 make_int4(static_cast<int>(r[j]), static_cast<int>(r[j + 1]),
                                           static_cast<int>(r[j + 2]), static_cast<int>(r[j + 3])));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.acc_empty[b]);
        named_barrier(1, 128);
        if (et == 0) mbar_arrive_remote_release(map_shared_rank(smem_u32(&bars.recv_full), 0u));
        continue;
      }
      if (role == 1 && first) {
        // first K half: the partner's partial must have landed
        ok = named_barrier_all(2, 128, mbar_wait_cluster(&bars.recv_full, 0, err));
        if (!ok) break;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < NT; c0 += C::kCh) {
        uint32_t r[C::kCh];
        load_acc(c0, r);
        if (role == 1 && first) {
          // plus the partner's partial (the other K half; 256 * acc stays
          // within int32 for K <= QVLA_MAX_K)
#pragma unroll
          for (int j = 0; j < C::kCh; j += 4) {
            const uint4 v = lds128(smem_u32(recv) + static_cast<uint32_t>((((c0 + j) >> 2) * kBM + row) * 16));
            r[j] += v.x;
            r[j + 1] += v.y;
            r[j + 2] += v.z;
            r[j + 3] += v.w;
          }
        }
        if (c0 + C::kCh >= NT) {
          // the accumulator may be reused once every warp has read it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.acc_empty[b]);
        }
        if (P.acc != nullptr) {
          if (nv) {
#pragma unroll
            for (int j = 0; j < C::kCh; ++j) {
              const int m = tr.m0 + c0 + j;
              if (m < P.M) P.acc[static_cast<size_t>(m) * P.N + n] = static_cast<int32_t>(r[j]) >> 8;
            }
          }
          continue;
        }
        __nv_bfloat16* ot = outs + (chunk % kOutSlots) * (C::kCh * kBM);
        // the store that last read this slot has finished reading it
        if (et == 0) bulk_wait_read<kOutSlots - 1>();
        named_barrier(1, 128);
        // the chunk's token scales as 16-byte shared loads (one per four
        // tokens, broadcast to the warp)
        float sxc[C::kCh];
#pragma unroll
        for (int j = 0; j < C::kCh; j += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(sx_s + c0 + j);
          sxc[j] = v4.x;
          sxc[j + 1] = v4.y;
          sxc[j + 2] = v4.z;
          sxc[j + 3] = v4.w;
        }
#pragma unroll
        for (int j = 0; j < C::kCh; ++j) {
          const int32_t a = static_cast<int32_t>(r[j]) >> 8;
          ot[j * kBM + row] = __float2bfloat16_rn(fmaf(sxc[j] * sw, static_cast<float>(a), bn));
        }
        fence_proxy_async_smem();
        named_barrier(1, 128);
        if (tma) {
          if (et == 0) tma_store_2d(&P.ty, ot, tr.n0, tr.m0 + c0);
        } else {
          // a tile cut by N with N % 8 != 0: plain stores, no box past N
          for (int e = et; e < C::kCh * kBM; e += 128) {
            const int c = e / kBM, nx = e % kBM;
            if (tr.n0 + nx < P.N && tr.m0 + c0 + c < P.M)
              P.y[static_cast<size_t>(tr.m0 + c0 + c) * P.ldy + tr.n0 + nx] = ot[c * kBM + nx];
          }
        }
        if (et == 0) bulk_commit();                // one group per chunk, maybe empty
        ++chunk;
      }
      // sx_s is rewritten for the next tile only after every thread is done
      // with this one
      named_barrier(1, 128);
    }
    if (et == 0) bulk_wait0();
    pdl_launch_dependents();
  }

  cta_sync();
  // phase 2: neither CTA of a pair leaves while the other may still reach
  // its shared memory
  if (batch.split) {
    if (!cluster_waited) cluster_wait();
    cluster_sync();
  }
  if (warp == 1) {
    __syncwarp();                  // lane 0 comes from the MMA loop
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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

bool encode(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t inner,
            uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
            CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promo) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  n = std::min(n, kMaxCtas);
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// A tile's cost in 128-wide K steps, plus a fixed share for its epilogue.
constexpr int kTileOverhead = 2;

// Longest-first list scheduling: each tile of `ids` (sorted by decreasing
// cost) to the CTA with the least work so far (ties: the lowest index),
// appended to that CTA's list.  Returns the largest load.
long long lpt(const std::vector<int>& ids, const std::vector<int>& cost,
              std::vector<long long>& load, std::vector<std::vector<int>>& lists) {
  using Load = std::pair<long long, int>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < static_cast<int>(load.size()); ++c) heap.push({load[c], c});
  for (int t : ids) {
    Load l = heap.top();
    heap.pop();
    lists[l.second].push_back(t);
    l.first += cost[t];
    load[l.second] = l.first;
    heap.push(l);
  }
  long long mx = 0;
  for (long long v : load) mx = std::max(mx, v);
  return mx;
}

// Deals the launch's tiles to the CTAs and writes the per-CTA lists; returns
// the number of CTAs.  With `pairs` > 0 (small token tiles, clusters of two
// available) the tiles much longer than the average load may be split over
// K between the two CTAs of a cluster: each half is the first tile of its
// CTA, rank 0 takes the first K half and the epilogue.  The split schedule is
// used when it shortens the longest list by more than a twentieth.
int schedule(Batch& b, int pairs) {
  const int T = b.tile_start[b.n];
  std::vector<int> ids(T), cost(T), units(T), nks(T);
  for (int p = 0; p < b.n; ++p)
    for (int t = b.tile_start[p]; t < b.tile_start[p + 1]; ++t) {
      units[t] = (b.p[p].K + 127) / 128;
      nks[t] = b.p[p].nks;
      cost[t] = units[t] + kTileOverhead;
    }
  for (int t = 0; t < T; ++t) ids[t] = t;
  std::stable_sort(ids.begin(), ids.end(), [&](int x, int y) { return cost[x] > cost[y]; });

  const int G1 = std::min(sm_count(), T);
  std::vector<long long> load1(G1, 0);
  std::vector<std::vector<int>> lists1(G1);
  const long long span1 = G1 > 0 ? lpt(ids, cost, load1, lists1) : 0;

  b.split = 0;
  std::vector<std::vector<int>> lists = lists1;
  std::vector<int8_t> role;
  if (pairs > 0 && T > 0) {
    const int G2 = 2 * pairs;
    long long total = 0;
    for (int t = 0; t < T; ++t) total += cost[t];
    std::vector<int> split, rest;
    for (int t : ids) {
      const bool long_tile = nks[t] >= 2 && 5 * cost[t] > 6 * (total / G2) &&
                             static_cast<int>(split.size()) < pairs;
      (long_tile ? split : rest).push_back(t);
    }
    if (!split.empty()) {
      std::vector<long long> load2(G2, 0);
      std::vector<std::vector<int>> lists2(G2);
      std::vector<int8_t> role2(G2, 0);
      for (size_t k = 0; k < split.size(); ++k) {
        const int t = split[k], h = 2 * (nks[t] / 2);       // 128-wide units of the first half
        lists2[2 * k].push_back(t);
        lists2[2 * k + 1].push_back(t);
        role2[2 * k] = 1;
        role2[2 * k + 1] = 2;
        load2[2 * k] = h + kTileOverhead + 1;
        load2[2 * k + 1] = (units[t] - h) + 1;
      }
      const long long span2 = lpt(rest, cost, load2, lists2);
      if (20 * span2 < 19 * span1) {
        b.split = 1;
        lists.swap(lists2);
        role.swap(role2);
      }
    }
  }
  // launch tile id -> problem | n-tile << 4 | m-tile << 19
  std::vector<uint32_t> packed(T);
  for (int p = 0; p < b.n; ++p)
    for (int t = b.tile_start[p]; t < b.tile_start[p + 1]; ++t) {
      const int local = t - b.tile_start[p] + b.p[p].tile_base;
      packed[t] = static_cast<uint32_t>(p) | static_cast<uint32_t>(local % b.p[p].tiles_n) << 4 |
                  static_cast<uint32_t>(local / b.p[p].tiles_n) << 19;
    }
  const int G = static_cast<int>(lists.size());
  int k = 0;
  for (int c = 0; c < G; ++c) {
    b.cta_begin[c] = static_cast<uint16_t>(k);
    b.role[c] = b.split ? role[c] : 0;
    for (int t : lists[c]) b.order[k++] = packed[t];
  }
  b.cta_begin[G] = static_cast<uint16_t>(k);
  return G;
}

// Clusters of two CTAs of this kernel the device holds at once (one CTA per
// SM), cached per device; 0 when that cannot be had.
template <int NT, bool kImage>
int cluster_pairs() {
  using C = Cfg<NT, kImage>;
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int c = cache[dev].load(std::memory_order_relaxed);
  if (c != 0) return c > 0 ? c : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * kMaxCtas, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, w4a4_gemm_kernel<NT, kImage>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  n = std::min(n, kMaxCtas / 2);
  cache[dev].store(n > 0 ? n : -1, std::memory_order_relaxed);
  return n;
}

template <int NT, bool kImage>
cudaError_t launch_batch(Batch& batch, cudaStream_t stream) {
  using C = Cfg<NT, kImage>;
  auto kern = w4a4_gemm_kernel<NT, kImage>;
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, [&]() {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (e != cudaSuccess) return e;
  const int G = schedule(batch, C::kSplit ? cluster_pairs<NT, kImage>() : 0);
  if (G == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (batch.split) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
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

// Fills problem slot `P` for the tiles of `g` from t0 on.
template <int NT, bool kImage>
bool fill_problem(Problem& P, const GemmArgs& g, int t0) {
  using C = Cfg<NT, kImage>;
  std::memset(&P, 0, sizeof(P));
  if (!encode(&P.tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.wq, g.K / 2, g.N, g.K / 2, kAPack, kBM,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return false;
  if (kImage) {
    if (!encode(&P.tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.xq8, g.K, g.M, g.K, 128, NT,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
      return false;
  } else {
    if (!encode(&P.tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.xq, g.K / 2, g.M, g.K / 2, 128, NT,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
      return false;
  }
  if (g.y != nullptr &&
      !encode(&P.ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.y, g.N, g.M,
              static_cast<uint64_t>(g.ldy) * 2, kBM, C::kCh, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_NONE))
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
  P.nks = (g.K + kKS - 1) / kKS;     // a ragged last stage reads zeros past K
  P.tile_base = t0;
  return true;
}

// All problems of one (token tile, activation form) group, in launches of at
// most kMaxBatch problems and kMaxTiles tiles (a problem with more tiles is
// cut into tile ranges).
template <int NT, bool kImage>
cudaError_t launch_group(const std::vector<const GemmArgs*>& gs, cudaStream_t stream) {
  Batch batch;
  std::memset(&batch, 0, sizeof(batch));
  int tiles = 0;
  auto flush = [&]() -> cudaError_t {
    if (batch.n == 0) return cudaSuccess;
    batch.tile_start[batch.n] = tiles;
    cudaError_t e = launch_batch<NT, kImage>(batch, stream);
    std::memset(&batch, 0, sizeof(batch));
    tiles = 0;
    return e;
  };
  for (const GemmArgs* g : gs) {
    // the packed tile coordinates hold 2^15 weight tiles and 2^13 token tiles
    if ((g->N + kBM - 1) / kBM > (1 << 15) || (g->M + NT - 1) / NT > (1 << 13))
      return cudaErrorInvalidValue;
    const int total = ((g->N + kBM - 1) / kBM) * ((g->M + NT - 1) / NT);
    for (int t0 = 0; t0 < total;) {
      if (batch.n == kMaxBatch || tiles == kMaxTiles) {
        cudaError_t e = flush();
        if (e != cudaSuccess) return e;
      }
      const int take = std::min(total - t0, kMaxTiles - tiles);
      if (!fill_problem<NT, kImage>(batch.p[batch.n], *g, t0)) return cudaErrorInvalidValue;
      batch.tile_start[batch.n] = tiles;
      ++batch.n;
      tiles += take;
      t0 += take;
    }
  }
  return flush();
}

int token_tile(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

template <bool kImage>
cudaError_t launch_form(const std::vector<const GemmArgs*>& v, cudaStream_t stream) {
  static const int kTiles[4] = {16, 32, 64, 128};
  for (int t : kTiles) {
    std::vector<const GemmArgs*> grp;
    for (const GemmArgs* g : v)
      if (token_tile(g->M) == t) grp.push_back(g);
    if (grp.empty()) continue;
    cudaError_t e;
    switch (t) {
      case 16: e = launch_group<16, kImage>(grp, stream); break;
      case 32: e = launch_group<32, kImage>(grp, stream); break;
      case 64: e = launch_group<64, kImage>(grp, stream); break;
      default: e = launch_group<128, kImage>(grp, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

bool encode_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t inner,
                   uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle) {
  return encode(map, dt, ptr, inner, outer, pitch, box_inner, box_outer, swizzle,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

cudaError_t launch_w4a4_gemm_batch(const GemmArgs* gs, int n, int /*split_k*/,
                                   cudaStream_t stream) {
  // linears whose activations come as the int8 image, and the packed rest
  std::vector<const GemmArgs*> img, pk;
  for (int i = 0; i < n; ++i)
    if (gs[i].M > 0) (gs[i].xq8 != nullptr ? img : pk).push_back(&gs[i]);
  cudaError_t e = launch_form<true>(img, stream);
  if (e == cudaSuccess) e = launch_form<false>(pk, stream);
  return e;
}

cudaError_t launch_w4a4_gemm(const GemmArgs& g, cudaStream_t stream) {
  return launch_w4a4_gemm_batch(&g, 1, g.split_k, stream);
}

}  // namespace qvla
