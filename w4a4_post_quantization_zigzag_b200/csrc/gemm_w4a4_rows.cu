// Persistent W4A4 GEMM for small token counts (M <= 64 tokens per linear),
// the regime of a DiT action chunk, where the layer is a stream of packed
// weights past a handful of activation rows:
//
//   acc[m,n] = sum_k q_x[m,k] q_w[n,k]                      (exact)
//   y[m,n]   = bf16( fp32(s_x[m] s_w[n]) * acc[m,n] + b[n] )
//
// ("Omega-QVLA: Nen VLA W4A4 tren Edge", section "Vi sao W4A4 kho hon
// W4A16?": both operands 4-bit, integer tensor cores.)
//
// Work split.  One CTA per SM for the whole batch of linears.  The weight rows
// of every linear are cut into granules of 8 rows (one 128-byte-swizzle atom);
// granules are ordered linear by linear, 128-row tile by tile, and every CTA
// takes a contiguous run whose weight bytes are an equal share of the total.
// A run is walked as items: the granules of one 128-row tile.  A tile cut
// between two CTAs is split by ROWS, not by K, so every output element is
// owned by exactly one CTA and no partial sums cross CTAs.  Rows of the MMA
// that an item does not own compute garbage that is never stored.
//
// Pipeline (14 warps):
//   warp 0      TMA producer: the whole run's weight tiles are requested into
//               L2 at start; then one ring stage per 256-wide K tile (the
//               item's weight rows as at most a few boxes of 128/64/32/16/8
//               rows, plus the NT code rows), continuing across items so the
//               ring never drains;
//   warps 2-9   unpack, two warpgroups taking alternate K tiles (so one
//               tile's load/convert/store latency overlaps the next): thread t
//               of a group owns weight row t (tensor-memory lane t) and turns
//               its row's 128 packed bytes into 256 int8 values 16*q written
//               to tensor memory (the MMA's A operand, which thus never touches
//               shared memory); the code rows go to a 128-byte swizzled
//               K-major shared-memory ring (the B operand);
//   warp 1      one thread issues tcgen05.mma kind::i8 (M = 128 weight rows,
//               N = NT tokens, K = 32) into one of two tensor-memory
//               accumulators, so an item's epilogue overlaps the next item;
//   warps 10-13 epilogue: tcgen05.ld of the whole accumulator, dequantisation
//               and bias; a whole 128-row tile leaves as one bf16 TMA tensor
//               store, a partial one as plain stores of its own rows.
// Every code group of 32 is laid out as its 16 even codes then its 16 odd
// codes in both operands (the same K order, so the dot product is unchanged);
// the accumulator holds 256*acc exactly and the epilogue shifts by 8.
//
// All waits are bounded (2 s) and flag QVLA_DEVERR_TIMEOUT instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "qvla_common.cuh"
#include "qvla_internal.h"

namespace qvla {
namespace {

constexpr int kBM = 128;               // weight rows per tile (UMMA M)
constexpr int kKP = 256;               // K per stage
constexpr int kRowP = kKP / 2;         // packed bytes per row per stage
constexpr int kGran = 8;               // weight rows per granule
constexpr int kGranPerTile = kBM / kGran;
constexpr int kBoxes = 5;              // weight boxes of 128, 64, 32, 16 and 8 rows
constexpr int kGroups = 2;             // unpack warpgroups (alternate K tiles)
constexpr int kThreads = 64 + kGroups * 128 + 128;
constexpr int kEpiWarp0 = 2 + kGroups * 4;
constexpr int kUS = 2 * kGroups;       // unpacked stages (A in tensor memory, B in smem)
constexpr int kMaxProblems = 16;
constexpr int kMaxCtas = 256;

template <int NT>
struct RCfg {
  static constexpr int kPStage = (kBM + NT) * kRowP;   // packed weights, then codes
  static constexpr int kBStage = NT * 2 * kRowP;       // unpacked codes: two 128-byte K halves
  static constexpr int kOTile = NT * kBM * 2;          // bf16 [NT tokens][128 channels]
  static constexpr int kFixed = kUS * kBStage + kOTile + 1024;
  static constexpr int kPSFit = (225 * 1024 - kFixed) / kPStage;
  static constexpr int kPS = kPSFit > 8 ? 8 : kPSFit;
  static constexpr int kSmem = kPS * kPStage + kFixed;
  static constexpr int kAccCols = NT < 32 ? 32 : NT;   // per accumulator
  static constexpr int kACol0 = 2 * kAccCols;          // first column of the A stages
  static constexpr int kTmemNeed = kACol0 + kUS * 64;
  static constexpr int kTmemCols = kTmemNeed <= 256 ? 256 : 512;
  static_assert(kPS >= 3, "ring too shallow");
  static_assert(kTmemNeed <= 512, "tensor memory");
  static_assert(kPStage % 1024 == 0 && kBStage % 1024 == 0, "swizzle atoms");
};

struct RBars {
  uint64_t full_p[8], empty_p[8];
  uint64_t full_u[kUS], empty_u[kUS];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
};

struct RProblem {
  CUtensorMap tw[kBoxes];         // packed weights [N][K/2], boxes 128 B x (128 >> i) rows
  CUtensorMap tx;                 // packed codes [M][K/2], box 128 B x NT rows
  CUtensorMap ty;                 // bf16 output [M][ldy], box 128 channels x NT tokens
  const float* s_x;
  const float* s_w;
  const float* bias;
  int32_t* acc;                   // int32 [M][N] output instead of y (tests)
  __nv_bfloat16* y;
  int M, N, K, ldy;
  int g0;                         // first granule of this linear in the launch
};

struct RBatch {
  int n;
  RProblem p[kMaxProblems];
  int cta_g0[kMaxCtas + 1];       // granule run of CTA c: [cta_g0[c], cta_g0[c+1])
};

// One item: granules [j0, j1) of 128-row tile `tile` of linear `p`.
struct Item {
  int p, tile, j0, j1;
};

// Next item of the run [g, g_end); advances g.
QVLA_DEVICE bool next_item(const RBatch& B, int& g, int g_end, Item& it) {
  if (g >= g_end) return false;
  int p = 0;
  while (p + 1 < B.n && g >= B.p[p + 1].g0) ++p;
  const int lg = g - B.p[p].g0;
  const int grans = (B.p[p].N + kGran - 1) / kGran;
  it.p = p;
  it.tile = lg / kGranPerTile;
  it.j0 = lg % kGranPerTile;
  const int end = min(min((it.tile + 1) * kGranPerTile, grans), lg + (g_end - g));
  it.j1 = end - it.tile * kGranPerTile;
  g += it.j1 - it.j0;
  return true;
}

// Rows [8 j0, 8 j1) of a tile as few TMA boxes as possible: at each step the
// largest box (128, 64, 32, 16, 8 rows) that starts at a multiple of its
// height and fits.  Calls f(box index, first row).
template <typename F>
QVLA_DEVICE void for_each_box(int j0, int j1, F&& f) {
  int r = j0 * kGran;
  const int r1 = j1 * kGran;
  while (r < r1) {
    int b = 0;
    while ((r % (kBM >> b)) != 0 || r + (kBM >> b) > r1) ++b;
    f(b, r);
    r += kBM >> b;
  }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_rows_kernel(const __grid_constant__ RBatch batch, unsigned int* err) {
  using C = RCfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ RBars bars;
  __shared__ __align__(16) float sx_s[2][NT];

  const int g_begin = batch.cta_g0[blockIdx.x];
  const int g_end = batch.cta_g0[blockIdx.x + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* const base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* const pstage = base;                                  // kPS packed stages
  uint8_t* const ustage = base + C::kPS * C::kPStage;            // kUS unpacked code stages
  uint8_t* const otile = ustage + kUS * C::kBStage;              // bf16 output tile

  if (tid == 0) {
    for (int s = 0; s < C::kPS; ++s) {
      mbar_init(&bars.full_p[s], 1);
      mbar_init(&bars.empty_p[s], 128);
    }
    for (int u = 0; u < kUS; ++u) {
      mbar_init(&bars.full_u[u], 128);
      mbar_init(&bars.empty_u[u], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], 1);
      mbar_init(&bars.acc_empty[b], 128);
    }
    mbar_init(&bars.drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();                  // tcgen05 alloc/ld/st/dealloc are warp-wide
    tmem_alloc(&bars.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // Stages before the first `kPS` get their weight rows before the wait
      // for the previous grid in the stream (weights do not depend on it) and
      // their code rows after it.  Then the rest of the run's weight tiles
      // are requested into L2 at once (after the first loads, which must not
      // queue behind them).
      int pre_p[8], pre_kt[8];
      int npre = 0;
      bool waited = false, ok = true;
      int i = 0, last_p = -1;
      int g = g_begin;
      Item it;
      while (ok && next_item(batch, g, g_end, it)) {
        const RProblem& P = batch.p[it.p];
        const int nkt = (P.K + kKP - 1) / kKP;
        const uint32_t wbytes = static_cast<uint32_t>((it.j1 - it.j0) * kGran * kRowP);
        const int n0 = it.tile * kBM;
        if (it.p != last_p) {        // descriptors of the linears this CTA touches
          for (int b = 0; b < kBoxes; ++b) tma_prefetch_desc(&P.tw[b]);
          tma_prefetch_desc(&P.tx);
          if (P.acc == nullptr) tma_prefetch_desc(&P.ty);
          last_p = it.p;
        }
        for (int kt = 0; kt < nkt; ++kt, ++i) {
          const int s = i % C::kPS;
          if (i >= C::kPS) {
            if (!waited) {
              pdl_wait();
              for (int q = 0; q < npre; ++q)
                tma_load_2d(pstage + q * C::kPStage + kBM * kRowP, &batch.p[pre_p[q]].tx,
                            &bars.full_p[q], pre_kt[q] * kRowP, 0);
              waited = true;
              // the remaining weight tiles of the run into L2
              int g2 = g_begin, i2 = 0;
              Item it2;
              while (next_item(batch, g2, g_end, it2)) {
                const RProblem& P2 = batch.p[it2.p];
                const int nkt2 = (P2.K + kKP - 1) / kKP;
                for (int k2 = 0; k2 < nkt2; ++k2, ++i2)
                  if (i2 >= C::kPS) tma_prefetch_l2_2d(&P2.tw[0], k2 * kRowP, it2.tile * kBM);
              }
            }
            ok = mbar_wait(&bars.empty_p[s], ((i / C::kPS) & 1) ^ 1u, err);
            if (!ok) break;
          }
          uint8_t* dst = pstage + s * C::kPStage;
          // a cut last tile is loaded as whole granules; rows past N are zero
          mbar_arrive_expect_tx(&bars.full_p[s], wbytes + NT * kRowP);
          for_each_box(it.j0, it.j1, [&](int b, int r) {
            tma_load_2d(dst + r * kRowP, &P.tw[b], &bars.full_p[s], kt * kRowP, n0 + r);
          });
          if (waited) {
            tma_load_2d(dst + kBM * kRowP, &P.tx, &bars.full_p[s], kt * kRowP, 0);
          } else {
            pre_p[npre] = it.p;
            pre_kt[npre] = kt;
            ++npre;
          }
        }
      }
      if (!waited) {
        pdl_wait();
        for (int q = 0; q < npre; ++q)
          tma_load_2d(pstage + q * C::kPStage + kBM * kRowP, &batch.p[pre_p[q]].tx,
                      &bars.full_p[q], pre_kt[q] * kRowP, 0);
      }
      // never leave with copies in flight
      for (int q = i - C::kPS < 0 ? 0 : i - C::kPS; q < i; ++q)
        mbar_wait(&bars.full_p[q % C::kPS], (q / C::kPS) & 1, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, NT);
      bool ok = true;
      int j = 0, item = 0;
      int g = g_begin;
      Item it;
      while (ok && next_item(batch, g, g_end, it)) {
        const int nkt = (batch.p[it.p].K + kKP - 1) / kKP;
        const int b = item & 1;
        if (item >= 2) {
          ok = mbar_wait(&bars.acc_empty[b], ((item >> 1) - 1) & 1, err);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t d = tmem + b * C::kAccCols;
        for (int kt = 0; kt < nkt; ++kt, ++j) {
          const int u = j % kUS;
          ok = mbar_wait(&bars.full_u[u], (j / kUS) & 1, err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_t = tmem + C::kACol0 + u * 64;
          const uint32_t b_s = smem_u32(ustage + u * C::kBStage);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // packed chunk kk: A columns [8kk, 8kk+8), B bytes [32(kk%4), +32)
            // of K half kk/4
            const uint64_t bd = smem_desc_kmajor_sw128(b_s + (kk >> 2) * NT * kRowP + 32 * (kk & 3));
            umma_i8_tmem_a(d, a_t + 8 * kk, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars.empty_u[u]);
        }
        if (!ok) break;
        umma_commit(&bars.acc_full[b]);
        ++item;
      }
      umma_commit(&bars.drain);
      mbar_wait(&bars.drain, 0, err);   // tensor memory is freed only after this
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------- unpack (kGroups warpgroups of 4)
    // Warpgroup `grp` takes the K tiles j with j % kGroups == grp, so the
    // latency of one tile's loads, conversions and stores overlaps the next.
    const int grp = (warp - 2) >> 2;
    const int wt = (warp - 2 - 4 * grp) * 32 + lane;   // 0..127 within the group
    const int row = (warp & 3) * 32 + lane;            // weight row = tensor-memory lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    constexpr int kBItems = NT * 8 / 128;              // code chunks per thread
    bool ok = true;
    int j = 0;
    int g = g_begin;
    Item it;
    while (ok && next_item(batch, g, g_end, it)) {
      const RProblem& P = batch.p[it.p];
      const int nkt = (P.K + kKP - 1) / kKP;
      const bool mine = row >= it.j0 * kGran && row < it.j1 * kGran;
      for (int kt = 0; kt < nkt; ++kt, ++j) {
        if (j % kGroups != grp) continue;
        const int s = j % C::kPS;
        // warp-uniform outcome: the tensor-memory stores below are warp-wide
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.full_p[s], (j / C::kPS) & 1, err));
        if (!ok) break;
        const uint32_t ps = smem_u32(pstage + s * C::kPStage);
        uint4 w[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          w[c] = mine ? lds128(ps + row * kRowP + ((c ^ (row & 7)) << 4))
                      : make_uint4(0u, 0u, 0u, 0u);
        // code chunk e: row e % NT, packed chunk e / NT (consecutive threads
        // take consecutive rows: conflict-free 128-byte-swizzled accesses)
        uint4 bw[kBItems];
#pragma unroll
        for (int k = 0; k < kBItems; ++k) {
          const int e = wt + k * 128;
          const int br = e % NT, c = e / NT;
          bw[k] = lds128(ps + (kBM + br) * kRowP + ((c ^ (br & 7)) << 4));
        }
        const int u = j % kUS;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars.empty_u[u], ((j / kUS) & 1) ^ 1u, err));
        if (!ok) break;
        tc_fence_after();
        // A: the row's 256 codes as 16*q int8, chunk c -> columns [8c, 8c+8)
        // (even codes of its four words, then odd codes)
        const uint32_t a_t = tmem + lane_base + C::kACol0 + u * 64;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t a[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = w[4 * hh + c];
            a[8 * c + 0] = (v.x << 4) & 0xF0F0F0F0u;
            a[8 * c + 1] = (v.y << 4) & 0xF0F0F0F0u;
            a[8 * c + 2] = (v.z << 4) & 0xF0F0F0F0u;
            a[8 * c + 3] = (v.w << 4) & 0xF0F0F0F0u;
            a[8 * c + 4] = v.x & 0xF0F0F0F0u;
            a[8 * c + 5] = v.y & 0xF0F0F0F0u;
            a[8 * c + 6] = v.z & 0xF0F0F0F0u;
            a[8 * c + 7] = v.w & 0xF0F0F0F0u;
          }
          tmem_st32(a_t + 32 * hh, a);
        }
        // B: packed chunk c of code row br -> K half c/4, unpacked chunks
        // 2(c%4) (even codes) and 2(c%4)+1 (odd codes), 128-byte swizzled
        const uint32_t us = smem_u32(ustage + u * C::kBStage);
#pragma unroll
        for (int k = 0; k < kBItems; ++k) {
          const int e = wt + k * 128;
          const int br = e % NT, c = e / NT;
          const int cl = c & 3;
          const uint4 v = bw[k];
          uint4 ev, od;
          ev.x = (v.x << 4) & 0xF0F0F0F0u;
          ev.y = (v.y << 4) & 0xF0F0F0F0u;
          ev.z = (v.z << 4) & 0xF0F0F0F0u;
          ev.w = (v.w << 4) & 0xF0F0F0F0u;
          od.x = v.x & 0xF0F0F0F0u;
          od.y = v.y & 0xF0F0F0F0u;
          od.z = v.z & 0xF0F0F0F0u;
          od.w = v.w & 0xF0F0F0F0u;
          const uint32_t rowp = us + (c >> 2) * NT * kRowP + br * kRowP;
          sts128(rowp + (((2 * cl) ^ (br & 7)) << 4), ev);
          sts128(rowp + (((2 * cl + 1) ^ (br & 7)) << 4), od);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars.full_u[u]);
        mbar_arrive(&bars.empty_p[s]);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int et = tid - 32 * kEpiWarp0;         // 0..127
    const int nl = (warp & 3) * 32 + lane;       // local output channel = tensor-memory lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t orow = smem_u32(otile) + nl * 2;   // column nl of the [NT][128] tile
    pdl_wait();                                  // s_x comes from the previous grid
    bool ok = true;
    int item = 0;
    int g = g_begin;
    Item it;
    while (ok && next_item(batch, g, g_end, it)) {
      const RProblem& P = batch.p[it.p];
      const int b = item & 1;
      const int n0 = it.tile * kBM;
      const int n = n0 + nl;
      const bool mine = nl >= it.j0 * kGran && nl < it.j1 * kGran && n < P.N;
      const bool to_y = P.acc == nullptr;
      // a whole tile (not cut by N) leaves through one TMA store; any other
      // item through plain stores of the rows it owns
      const bool whole = it.j0 == 0 && it.j1 == kGranPerTile && n0 + kBM <= P.N;
      const float sw = (to_y && mine) ? __ldg(P.s_w + n) : 0.f;
      const float bn = (to_y && mine && P.bias != nullptr) ? __ldg(P.bias + n) : 0.f;
      if (to_y)
        for (int c = et; c < NT; c += 128) sx_s[b][c] = c < P.M ? __ldg(P.s_x + c) : 0.f;
      if (et == 0) bulk_wait_read0();            // the previous item's store has read otile
      named_barrier(1, 128);
      // one outcome for all 128 threads: they share named barrier 1
      ok = named_barrier_all(1, 128, mbar_wait(&bars.acc_full[b], (item >> 1) & 1, err));
      if (!ok) break;
      __syncwarp();                // converged warp for the warp-wide loads
      tc_fence_after();
      const uint32_t tb = tmem + lane_base + b * C::kAccCols;
      uint32_t r[NT];
#pragma unroll
      for (int c0 = 0; c0 < NT; c0 += 16)
        tmem_ld16(tb + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[c0]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[b]);           // the accumulator may be reused
      if (mine) {
        if (!to_y) {
#pragma unroll
          for (int c = 0; c < NT; ++c)
            if (c < P.M) P.acc[static_cast<size_t>(c) * P.N + n] = static_cast<int32_t>(r[c]) >> 8;
        } else {
#pragma unroll
          for (int c = 0; c < NT; ++c) {
            const int32_t a = static_cast<int32_t>(r[c]) >> 8;
            const __nv_bfloat16 v =
                __float2bfloat16_rn(fmaf(sx_s[b][c] * sw, static_cast<float>(a), bn));
            if (whole)
              sts16(orow + c * kBM * 2, __bfloat16_as_ushort(v));
            else if (c < P.M)
              P.y[static_cast<size_t>(c) * P.ldy + n] = v;
          }
        }
      }
      if (to_y && whole) {
        fence_proxy_async_smem();
        named_barrier(1, 128);
        if (et == 0) {
          tma_store_2d(&P.ty, otile, n0, 0);
          bulk_commit();
        }
      }
      ++item;
    }
    pdl_launch_dependents();
    if (et == 0) bulk_wait0();
    tc_fence_before();
  }

  cta_sync();
  if (warp == 1) {
    __syncwarp();                  // lane 0 comes from the MMA loop
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

int sm_count() {
  static int counts[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (counts[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
      c = 148;
    counts[dev] = c;
  }
  return counts[dev];
}

template <int NT>
cudaError_t launch_rows_nt(const GemmArgs* const* gs, int n, cudaStream_t stream) {
  using C = RCfg<NT>;
  RBatch batch;
  std::memset(&batch, 0, sizeof(batch));
  batch.n = n;
  int g = 0;
  for (int i = 0; i < n; ++i) {
    const GemmArgs& a = *gs[i];
    RProblem& P = batch.p[i];
    const uint64_t kb = static_cast<uint64_t>(a.K / 2);
    for (int b = 0; b < kBoxes; ++b)
      if (!encode_map_2d(&P.tw[b], CU_TENSOR_MAP_DATA_TYPE_UINT8, a.wq, kb, a.N, kb, kRowP,
                         kBM >> b, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!encode_map_2d(&P.tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.xq, kb, a.M, kb, kRowP, NT,
                       CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (a.y != nullptr &&
        !encode_map_2d(&P.ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, a.N, a.M,
                       static_cast<uint64_t>(a.ldy) * 2, kBM, NT, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    P.s_x = a.s_x;
    P.s_w = a.w_scale;
    P.bias = a.bias;
    P.acc = a.y == nullptr ? a.acc : nullptr;
    P.y = static_cast<__nv_bfloat16*>(a.y);
    P.M = a.M;
    P.N = a.N;
    P.K = a.K;
    P.ldy = a.ldy;
    P.g0 = g;
    g += (a.N + kGran - 1) / kGran;
  }
  const int g_total = g;
  const int G = std::min(std::min(sm_count(), kMaxCtas), g_total);
  // Cost of a granule: its K tiles x (8 weight rows); the first granule of a
  // tile also carries the tile's per-K-tile overhead (the NT code rows to
  // load and unpack), counted as NT/2 weight rows.  CTA c starts at the first
  // granule whose cumulative cost reaches c/G of the total.
  std::vector<long long> cum(static_cast<size_t>(g_total) + 1, 0);
  for (int i = 0, gg = 0; i < n; ++i) {
    const int grans = (gs[i]->N + kGran - 1) / kGran;
    const long long nkt = (gs[i]->K + kKP - 1) / kKP;
    for (int q = 0; q < grans; ++q, ++gg)
      cum[gg + 1] = cum[gg] + nkt * (kGran + (q % kGranPerTile == 0 ? NT / 2 : 0));
  }
  const long long total = cum[g_total];
  batch.cta_g0[0] = 0;
  for (int c = 1; c < G; ++c) {
    const long long target = (total * c + G - 1) / G;
    const int gg = static_cast<int>(std::lower_bound(cum.begin(), cum.end(), target) - cum.begin());
    batch.cta_g0[c] = std::max(std::min(gg, g_total), batch.cta_g0[c - 1]);
  }
  batch.cta_g0[G] = g_total;
  auto kern = w4a4_gemm_rows_kernel<NT>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, batch, device_error_word());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a4_gemm_rows(const GemmArgs* const* gs, int n, int nt, cudaStream_t stream) {
  for (int i0 = 0; i0 < n; i0 += kMaxProblems) {
    const int m = std::min(kMaxProblems, n - i0);
    cudaError_t e;
    switch (nt) {
      case 16: e = launch_rows_nt<16>(gs + i0, m, stream); break;
      case 32: e = launch_rows_nt<32>(gs + i0, m, stream); break;
      case 64: e = launch_rows_nt<64>(gs + i0, m, stream); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qvla
