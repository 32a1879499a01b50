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
#include <cstdlib>
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

// The same code as quant_code(v, s, ...), i.e. clamp(rint(fp32(v / s))), with
// the IEEE division replaced by v * rs (rs = fp32(1 / s)) wherever that cannot
// change the rounding: the product is within 2^-19 of the exact quotient for
// |quotient| < 16 (two roundings of 2^-24 relative), so unless it lies within
// 2^-18 of a half-integer both round to the same integer; near a half-integer
// (about 1 element in 10^5) the exact division decides.  Quotients of 16 or
// more clamp either way.
// Kept out of line so the compiler cannot hoist the rare exact division into
// the common path.
__device__ __noinline__ float exact_rint_quotient(float v, float s) { return rintf(__fdiv_rn(v, s)); }

QVLA_DEVICE int quant_code_fast(float v, float s, float rs, int qmin, int qmax) {
  if (s == 0.f) return 0;
  if (rs == 0.f) return quant_code(v, s, qmin, qmax);
  const float q = v * rs;
  float r = rintf(q);
  if (fabsf(fabsf(q - r) - 0.5f) < 3.814697265625e-06f) r = exact_rint_quotient(v, s);
  r = fminf(fmaxf(r, static_cast<float>(qmin)), static_cast<float>(qmax));
  return static_cast<int>(r);
}

// Two fp32 lanes in one 64-bit register, for the paired FMA (sm_100).
QVLA_DEVICE uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
QVLA_DEVICE void f2split(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
QVLA_DEVICE uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
QVLA_DEVICE float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// One 32-byte store (sm_100); the address must be 32-byte aligned.
QVLA_DEVICE void st_global_v8(void* p, uint4 a, uint4 b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y),
               "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}
QVLA_DEVICE float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 4-bit codes of N consecutive values, packed two per byte (value 2k in the
// low nibble of byte k) into N/8 32-bit words: the same codes as
// quant_code(v, s, -8, 7) = clamp(rint(fp32(v / s)), -8, 7), as straight-line
// FMA-pipe code (so the independent elements overlap) with the rare elements
// near a rounding boundary redone by the IEEE division afterwards.  With
// a = fp32(1 / fp32(15 s)) (quant_recip15) and c8 = fp32(8 / 15):
//   * x = sat(fma(v, a, c8)) is (v/s + 8) / 15 clamped to [0, 1]: the
//     saturation is the clamp to [-8, 7] (clamping before rounding gives the
//     code of clamping after it: integer bounds, monotone rounding; NaN
//     saturates to 0, code -8, as the clamp of NaN gives);
//   * e = fp32(15 x + 1.5 * 2^23) - 1.5 * 2^23 is the offset code c + 8 =
//     rint(15 x) in [0, 15] (one rounding of the exact product, in a binade
//     of unit spacing: ties to even, as rint);
//   * |15 x - (fp32(v / s) + 8)| <= 2^-18.8 (2^-23 relative error in a, two
//     2^-25 roundings in x, 2^-22 in the IEEE quotient), so unless
//     d = 15 x - e (formed by one FMA) lies within 2^-18 of +-1/2 both round
//     to the same integer; near +-1/2 (about 1 element in 10^5) the exact
//     division decides;
//   * four offset codes go into one float as 2^23 + sum_j e_j 16^j, every
//     partial sum an integer in [2^23, 2^24), so its low 16 mantissa bits are
//     the four nibbles; XOR 8 turns an offset nibble into the 4-bit two's
//     complement of c.
// Values 8k + j and 8k + 4 + j share one paired FMA (the two packed floats of
// a word are built side by side).
constexpr float kNearHalf = 0.499996185302734375f;   // 1/2 - 2^-18
constexpr float kRound = 12582912.0f;                // 1.5 * 2^23
constexpr float kC8 = 0.533333361148834228515625f;   // fp32(8 / 15)

template <int N>
QVLA_DEVICE void quant_pack(const float (&v)[N], float s, float a15, uint32_t (&w)[N / 8]) {
  static_assert(N % 8 == 0 && N <= 32, "8..32 values");
  float ne[N];                                       // -(c + 8)
  if (s == 0.f) {
#pragma unroll
    for (int i = 0; i < N; ++i) ne[i] = -8.f;
  } else if (a15 == 0.f) {
#pragma unroll
    for (int i = 0; i < N; ++i) ne[i] = -(fminf(fmaxf(exact_rint_quotient(v[i], s), -8.f), 7.f) + 8.f);
  } else {
    const uint64_t k15 = f2(15.f, 15.f), kR = f2(kRound, kRound), kM1 = f2(-1.f, -1.f);
    float dmax = 0.f;
#pragma unroll
    for (int k = 0; k < N / 8; ++k) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i0 = 8 * k + j, i1 = i0 + 4;
        const uint64_t x = f2(fma_sat(v[i0], a15, kC8), fma_sat(v[i1], a15, kC8));
        const uint64_t m = ffma2(x, k15, kR);         // 1.5 * 2^23 + e
        const uint64_t n = ffma2(m, kM1, kR);         // -e, exact
        float d0, d1;
        f2split(ffma2(x, k15, n), d0, d1);            // 15 x - e, exact
        dmax = max3(dmax, fabsf(d0), fabsf(d1));
        f2split(n, ne[i0], ne[i1]);
      }
    }
    if (dmax > kNearHalf) {
#pragma unroll
      for (int i = 0; i < N; ++i)
        if (fabsf(fmaf(fma_sat(v[i], a15, kC8), 15.f, ne[i])) > kNearHalf)
          ne[i] = -(fminf(fmaxf(exact_rint_quotient(v[i], s), -8.f), 7.f) + 8.f);
    }
  }
  const uint64_t k23 = f2(8388608.0f, 8388608.0f);    // 2^23
#pragma unroll
  for (int k = 0; k < N / 8; ++k) {
    const float* n = ne + 8 * k;
    uint64_t h = ffma2(f2(n[0], n[4]), f2(-1.f, -1.f), k23);
    h = ffma2(f2(n[1], n[5]), f2(-16.f, -16.f), h);
    h = ffma2(f2(n[2], n[6]), f2(-256.f, -256.f), h);
    h = ffma2(f2(n[3], n[7]), f2(-4096.f, -4096.f), h);
    float h0, h1;
    f2split(h, h0, h1);
    w[k] = __byte_perm(__float_as_uint(h0), __float_as_uint(h1), 0x5410) ^ 0x88888888u;
  }
}

// fp32(1 / fp32(15 s)) for quant_pack, or 0 to force the exact path: s == 0,
// or 15 s or its reciprocal outside the normal range (the error bound of
// quant_pack takes both roundings as relative).
QVLA_DEVICE float quant_recip15(float s) {
  const float t = fabsf(15.f * s);
  if (!(t >= 1.17549435e-38f && t <= 4.2535296e37f)) return 0.f;   // [2^-126, 2^125]; NaN too
  return __frcp_rn(15.f * s);
}

// fp32(1 / s) for quant_code_fast, or 0 to force the exact path (s == 0 or a
// reciprocal that overflows).
QVLA_DEVICE float quant_recip(float s) {
  if (s == 0.f) return 0.f;
  const float rs = __frcp_rn(s);
  return isfinite(rs) ? rs : 0.f;
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
  CUtensorMap txp;            // permuted copy of x (tensor-core path with scratch)
  const void* x;
  const int32_t* perm;
  const float* rot;
  const uint16_t* rot_tc;
  const float* table;
  const int32_t* step_dev;
  uint8_t* xq;
  int8_t* xq8;                // int8 image of the codes (tensor-core route), or null
  float* s_x;
  float* xr_out;
  int M, ldx, K, T, Lcount, step_host, layer;
  int gx;                     // token tiles
  int bpc;                    // rotation blocks per CTA
  int a_rows;                 // rows of the permuted-x TMA box (tokens, <= 128)
  // DYNAMIC as two launches (ActBatch::phase 1 and 2): the row maxima of
  // every CTA's blocks, [ngroups][M] as fp32 bits
  unsigned int* amax;
  int ngroups;
};
struct ActBatch {
  int n;
  // DYNAMIC only.  0: both passes in one launch, the row maximum reduced over
  // a cluster along the blocks (grid y);  1: the maximum pass alone, each
  // CTA's row maxima to ActProblem::amax;  2: the quantising pass alone,
  // the scale from the maxima phase 1 wrote.  Phases 1 and 2 take no cluster.
  int phase;
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
  // no R_SVD blocks: the Hadamard-only rotation (R_SVD = I), x'_B = H x_B
  const bool hadamard_only = rot == nullptr;
  const int nchunks = hadamard_only ? 0 : nbc * G::NCH;
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
  cta_sync();   // perm_s visible

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
    // 2. dense product over R chunks (the gathered inputs themselves when
    // R_SVD = I)
    float acc[TPT][2];
#pragma unroll
    for (int u = 0; u < TPT; ++u) acc[u][0] = acc[u][1] = 0.f;
    if (hadamard_only) {
      cta_sync();   // the gather is complete
#pragma unroll
      for (int u = 0; u < TPT; ++u) {
        acc[u][0] = xg[(2 * jp) * TT + tg * TPT + u];
        acc[u][1] = xg[(2 * jp + 1) * TT + tg * TPT + u];
      }
      cta_sync();   // every thread has read its inputs before they are overwritten
    }
    for (int ch = 0; ch < (hadamard_only ? 0 : G::NCH); ++ch) {
      const int g = bl * G::NCH + ch;
      if (g + 1 < nchunks) {
        issue_chunk(g + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      cta_sync();
      const float* Rc = rbuf + (g & 1) * G::kChunkFloats;
#pragma unroll 4
      for (int ii = 0; ii < G::RCH; ++ii) {
        const float2 r = *reinterpret_cast<const float2*>(Rc + ii * BS + 2 * jp);
        const float* xrow = xg + (ch * G::RCH + ii) * TT + tg * TPT;
        // the thread's TPT tokens in as few (warp-broadcast) loads as possible
        float xv[TPT];
        if constexpr (TPT % 4 == 0) {
#pragma unroll
          for (int u = 0; u < TPT; u += 4) {
            const float4 q = *reinterpret_cast<const float4*>(xrow + u);
            xv[u] = q.x; xv[u + 1] = q.y; xv[u + 2] = q.z; xv[u + 3] = q.w;
          }
        } else if constexpr (TPT % 2 == 0) {
#pragma unroll
          for (int u = 0; u < TPT; u += 2) {
            const float2 q = *reinterpret_cast<const float2*>(xrow + u);
            xv[u] = q.x; xv[u + 1] = q.y;
          }
        } else {
#pragma unroll
          for (int u = 0; u < TPT; ++u) xv[u] = xrow[u];
        }
#pragma unroll
        for (int u = 0; u < TPT; ++u) {
          acc[u][0] = fmaf(r.x, xv[u], acc[u][0]);
          acc[u][1] = fmaf(r.y, xv[u], acc[u][1]);
        }
      }
      cta_sync();   // chunk buffer (g & 1) may be refilled next
    }
    // 3. stage the products token-major (over the gather buffer)
#pragma unroll
    for (int u = 0; u < TPT; ++u)
      *reinterpret_cast<float2*>(xg + (tg * TPT + u) * BS + 2 * jp) =
          make_float2(acc[u][0], acc[u][1]);
    cta_sync();
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
        const float rs = quant_recip(s_tab);
#pragma unroll
        for (int c = 0; c < C; ++c)
          store_codes32(dst + 16 * c, quant_code_fast(v[c], s_tab, rs, -8, 7), lane);
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
    cta_sync();   // gather buffer reused by the next block
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
  cta_sync();
  if (blockIdx.y == 0 && tid < ntok) s_x[m0 + tid] = scale_s[tid];
  const int nch = nbc * BS;                    // channels held by this CTA (multiple of 32)
  for (int t = warp; t < ntok; t += kWarps) {
    const float s = scale_s[t];
    const float a15 = quant_recip15(s);
    uint8_t* dst = xq + static_cast<size_t>(m0 + t) * (K / 2) + (B0 * BS) / 2;
    for (int c0 = 0; c0 < nch; c0 += 256) {
      const int k = c0 + 8 * lane;            // 8 channels -> 4 bytes per lane
      if (k < nch) {
        const float4 a = *reinterpret_cast<const float4*>(keep + t * kpitch + k);
        const float4 b = *reinterpret_cast<const float4*>(keep + t * kpitch + k + 4);
        const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t w[1];
        quant_pack<8>(f, s, a15, w);
        *reinterpret_cast<uint32_t*>(dst + k / 2) = w[0];
      }
    }
  }
  if (cs > 1) cluster_wait();                  // peers finished reading our maxima
}

// ===========================================================================
// Composite CUDA-core path (block 64, TABLE and rotate-only modes, a linear
// that carries the tensor-core image of R_B, input the tensor-core route does
// not take: fp32).
//
// x'_B = x_B . R_B with the composite R_B = R_SVD,B . H_b itself: the image's
// three bf16 parts are summed in fp32 ((hi + mid) + lo, within one fp32 ulp
// of R_B), so no Walsh-Hadamard step follows the product.  One CTA = 32
// tokens x one rotation block at a time, 128 threads, each holding a
// 4-channel x 4-token register tile (16 fp32 FMA per two 16-byte shared
// loads); codes are formed and stored straight from the registers.
// ===========================================================================
constexpr int kCThreads = 128;
constexpr int kCBS = 64;
constexpr int kCTT = 32;

QVLA_DEVICE void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}

template <typename Tin, int MODE>
__global__ void __launch_bounds__(kCThreads)
    rotq_comp_kernel(const __grid_constant__ ActBatch batch, unsigned int* err) {
  __shared__ __align__(16) float comp[kCBS * kCBS];     // R_B[i][j], input-major, swizzled
  __shared__ __align__(16) float xg[kCBS * kCTT];       // x[t][perm[i]] at [i][t]
  __shared__ int32_t perm_s[kCBS];

  int pi = 0;
  while (pi + 1 < batch.n && static_cast<int>(blockIdx.x) >= batch.cta_start[pi + 1]) ++pi;
  const ActProblem& P = batch.p[pi];
  const Tin* __restrict__ x = static_cast<const Tin*>(P.x);
  const int M = P.M, ldx = P.ldx, K = P.K;
  const int local = static_cast<int>(blockIdx.x) - batch.cta_start[pi];
  const int tile = local % P.gx;
  const int group = local / P.gx;
  const int m0 = tile * kCTT;
  const int ntok = min(kCTT, M - m0);
  const int nb = K / kCBS;
  const int B0 = group * P.bpc;
  const int nbc = max(0, min(P.bpc, nb - B0));

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j0 = (warp & 1) * 32 + (lane & 7) * 4;      // four output channels
  const int t0 = (warp >> 1) * 16 + (lane >> 3) * 4;    // four tokens

  float s_tab = 0.f;
  for (int bl = 0; bl < nbc; ++bl) {
    const int B = B0 + bl;
    // 1. R_B from the image (weights: for the first block this runs before
    // the wait on the previous kernel).  A 16-byte chunk q of part sp holds
    // inputs 8c..8c+7 of output j = q / 8, c = (q % 8) ^ (j % 8); a warp
    // reads 32 consecutive chunks.  R_B[i][j] lands in row i at the 4-float
    // granule (j / 4) ^ (i / 8 % 8): the transposing stores of a warp and the
    // product's 16-byte reads both hit 32 different banks.
    const uint4* img = reinterpret_cast<const uint4*>(P.rot_tc + static_cast<size_t>(B) * 3 * kCBS * kCBS);
#pragma unroll
    for (int q = tid; q < kCBS * 8; q += kCThreads) {
      const int j = q >> 3, c = (q & 7) ^ (j & 7);
      const int col = 4 * ((j >> 2) ^ c) + (j & 3);
      const uint4 h = __ldg(img + q), m = __ldg(img + 512 + q), l = __ldg(img + 1024 + q);
      const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, mw[4] = {m.x, m.y, m.z, m.w},
                     lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float h0, h1, m0f, m1f, l0, l1;
        bf16x2_to_f32(hw[k], h0, h1);
        bf16x2_to_f32(mw[k], m0f, m1f);
        bf16x2_to_f32(lw[k], l0, l1);
        comp[(8 * c + 2 * k) * kCBS + col] = (h0 + m0f) + l0;
        comp[(8 * c + 2 * k + 1) * kCBS + col] = (h1 + m1f) + l1;
      }
    }
    if (tid < kCBS) perm_s[tid] = __ldg(P.perm + static_cast<size_t>(B) * kCBS + tid);
    if (bl == 0) {
      pdl_wait();
      pdl_launch_dependents();
      if (MODE == kTable)
        s_tab = table_scale(P.table, P.T, P.Lcount, P.step_dev, P.step_host, P.layer, err);
    }
    cta_sync();   // perm_s and comp complete
    // 2. gather the block's inputs, token-contiguous
#pragma unroll
    for (int e = tid; e < kCBS * kCTT; e += kCThreads) {
      const int i = e / kCTT, t = e % kCTT;
      const int p = perm_s[i];
      float v = 0.f;
      if (t < ntok && static_cast<unsigned>(p) < static_cast<unsigned>(K))
        v = load_x(x + static_cast<size_t>(m0 + t) * ldx + p);
      xg[e] = v;
    }
    cta_sync();
    // 3. acc[u][c] = sum_i x[t0 + u][i] R_B[i][j0 + c], in input order
    float acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[u][c] = 0.f;
#pragma unroll 8
    for (int i = 0; i < kCBS; ++i) {
      const float4 r = *reinterpret_cast<const float4*>(comp + i * kCBS + 4 * ((j0 >> 2) ^ ((i >> 3) & 7)));
      const float4 xv = *reinterpret_cast<const float4*>(xg + i * kCTT + t0);
      const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[u][0] = fmaf(xs[u], r.x, acc[u][0]);
        acc[u][1] = fmaf(xs[u], r.y, acc[u][1]);
        acc[u][2] = fmaf(xs[u], r.z, acc[u][2]);
        acc[u][3] = fmaf(xs[u], r.w, acc[u][3]);
      }
    }
    // 4. codes (or rotated values) straight from the registers
    if (MODE == kRotateOnly) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (t0 + u < ntok)
          *reinterpret_cast<float4*>(P.xr_out + static_cast<size_t>(m0 + t0 + u) * K + B * kCBS + j0) =
              make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    } else {
      const float rs = quant_recip(s_tab);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (t0 + u >= ntok) continue;
        uint32_t w = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          w |= static_cast<uint32_t>(quant_code_fast(acc[u][c], s_tab, rs, -8, 7) & 15) << (4 * c);
        *reinterpret_cast<uint16_t*>(P.xq + static_cast<size_t>(m0 + t0 + u) * (K / 2) + (B * kCBS + j0) / 2) =
            static_cast<uint16_t>(w);
      }
    }
    cta_sync();   // comp, xg and perm_s are refilled for the next block
  }
  if (MODE == kTable && group == 0 && tid < ntok) P.s_x[m0 + tid] = s_tab;
}

// ===========================================================================
// Tensor-core path (bf16 input, block 64 or 128).
//
// The block rotation is one dense product x'_B = x_B . R_B with the composite
// R_B = R_SVD,B . H_b, on tcgen05 (kind::f16, fp32 accumulation in tensor
// memory).  bf16 activations are exact in bf16; R_B is carried as three bf16
// parts (hi + mid + lo, pack time), so the product has ~fp32 accuracy.
// Per CTA: a tile of 128 tokens (the UMMA M dimension) and a run of blocks.
// With the permuted copy of x (the usual route):
//   warp 0      loads the A tiles by TMA and bulk-copies the R_B parts
//               (pre-swizzled images) into a ring
//   warp 1      issues the MMAs (3 parts x b/16 K-steps per block)
//   warps 2-9   read the accumulator and quantise: one token per thread,
//               warps 2-5 the first half of the block's columns, 6-9 the rest
// Without it, warps 2-5 gather x[m, perm[B*b + i]] into the A tile instead
// and warps 6-9 take every column.
// DYNAMIC mode runs the blocks twice: pass 0 takes each token's max |x'|
// (reduced over the cluster that shares the row), pass 1 quantises.
// ===========================================================================
using EncodeTiledFnR = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
constexpr int kTM = 128;

// kLat: the latency configuration for launches whose (token tile, block)
// pairs fit three CTAs per SM: six warps, one block per CTA, rings of two A
// tiles and one R_B, 57 KB of shared memory (block 64).
template <int BS, bool kLat = false>
struct TcCfg {
  static constexpr int kThreads = kLat ? 192 : 320;
  static constexpr int kAStage = kTM * BS * 2;          // bf16 A tile
  static constexpr int kRStage = BS * BS * 2;           // one bf16 part of R_B^T
  static constexpr int kAS = kLat ? 2 : BS == 64 ? 3 : 2;   // A tiles in flight
  static constexpr int kRS = kLat ? 3 : BS == 64 ? 6 : 4;
  static constexpr int kTmemCols = 2 * BS;              // double-buffered fp32 accumulator
  static constexpr int kSmem = kAS * kAStage + kRS * kRStage + 1024;
};

struct TcBars {
  uint64_t full_a[3], empty_a[3], full_r[6], empty_r[6], acc_full[2], acc_empty[2];
  uint32_t tmem;
};
static_assert(TcCfg<64>::kAS <= 3 && TcCfg<128>::kAS <= 3 && TcCfg<64>::kRS <= 6 &&
                  TcCfg<128>::kRS <= 6 && TcCfg<64, true>::kRS >= 3, "ring barriers");

QVLA_DEVICE void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Block 64 runs two CTAs per SM (three in the latency configuration; the
// grid is sized for that): the register budget must let them share the
// register file.
template <int BS, int MODE, bool kTmaA, bool kLat>
__global__ void __launch_bounds__(TcCfg<BS, kLat>::kThreads, kLat ? 3 : BS == 64 ? 2 : 1)
    rotq_tc_kernel(const __grid_constant__ ActBatch batch, unsigned int* err) {
  using C = TcCfg<BS, kLat>;
  // epilogue warps: 6-9, or 2-9 in two column halves when the A tiles come
  // by TMA and the gather warps are free; 2-5 in the latency configuration
  constexpr int kWarps = C::kThreads / 32;
  constexpr int kEpiWarps = (kTmaA && !kLat) ? 8 : 4;
  constexpr int kFirstEpi = kWarps - kEpiWarps;
  static_assert(!kLat || kTmaA, "the latency configuration loads A by TMA");
  constexpr int kHalves = kEpiWarps / 4;
  extern __shared__ uint8_t smem_raw[];
  __shared__ TcBars bars;
  __shared__ unsigned int amax_s[kTM];

  int pi = 0;
  while (pi + 1 < batch.n && static_cast<int>(blockIdx.x) >= batch.cta_start[pi + 1]) ++pi;
  const ActProblem& P = batch.p[pi];
  const __nv_bfloat16* __restrict__ x = static_cast<const __nv_bfloat16*>(P.x);
  const int M = P.M, ldx = P.ldx, K = P.K;
  const int local = static_cast<int>(blockIdx.x) - batch.cta_start[pi];
  const int tile = local % P.gx;
  const int phase = MODE == kDynamic ? batch.phase : 0;
  const int group = MODE == kDynamic && phase == 0 ? static_cast<int>(blockIdx.y) : local / P.gx;
  const int m0 = tile * kTM;
  const int ntok = min(kTM, M - m0);
  const int nb = K / BS;
  const int B0 = group * P.bpc;
  const int nbc = max(0, min(P.bpc, nb - B0));
  const int passes = MODE == kDynamic && phase == 0 ? 2 : 1;
  const int W = passes * nbc;                  // work items: (pass, block)
  const int cs = MODE == kDynamic && phase == 0 ? static_cast<int>(gridDim.y) : 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* const base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* const astage = base;
  uint8_t* const rstage = base + C::kAS * C::kAStage;

  if (tid == 0) {
    for (int i = 0; i < C::kAS; ++i) {
      mbar_init(&bars.full_a[i], kTmaA ? 1 : 128);
      mbar_init(&bars.empty_a[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.acc_full[i], 1);
      mbar_init(&bars.acc_empty[i], 32 * kEpiWarps);
    }
    for (int i = 0; i < C::kRS; ++i) {
      mbar_init(&bars.full_r[i], 1);
      mbar_init(&bars.empty_r[i], 1);
    }
    fence_mbar_init();
  }
  if (tid < kTM) amax_s[tid] = 0u;
  if (warp == 1) {
    __syncwarp();                  // tcgen05 alloc/ld/dealloc are warp-wide
    tmem_alloc(&bars.tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem = bars.tmem;
  const bool epi = warp >= kFirstEpi;
  // cluster barrier phase 1 ("row maxima published"): threads that are not in
  // the epilogue arrive once their pass-0 work is issued, so the epilogue's
  // wait never depends on work that waits for the epilogue
  bool arrived1 = false;

  if (warp == 0 && kTmaA) {
    // ------------------------------------- A tiles (permuted x) and R_B parts
    if (lane == 0) {
      auto issue_r = [&](int u) -> bool {
        const int rr = u % C::kRS, B = B0 + (u / 3) % nbc;
        if (!mbar_wait(&bars.empty_r[rr], ((u / C::kRS) & 1) ^ 1u, err)) return false;
        mbar_arrive_expect_tx(&bars.full_r[rr], C::kRStage);
        bulk_copy_g2s(rstage + rr * C::kRStage,
                      P.rot_tc + (static_cast<size_t>(B) * 3 + u % 3) * BS * BS, C::kRStage,
                      &bars.full_r[rr]);
        return true;
      };
      const int U = 3 * W;
      int ur = 0, issued = 0;
      bool ok = true;
      // the parts that fit the ring go out before the wait for the permuted copy
      while (ok && ur < min(U, C::kRS)) ok = issue_r(ur++) ;
      pdl_wait();
      for (int w = 0; ok && w < W; ++w) {
        const int B = B0 + w % nbc, as = w % C::kAS;
        if (!mbar_wait(&bars.empty_a[as], ((w / C::kAS) & 1) ^ 1u, err)) break;
        // a box of a_rows tokens (fewer than 128 for a short batch: the
        // MMA's rows past them hold stale values, and so do only its result
        // rows past them, which nothing reads)
        mbar_arrive_expect_tx(&bars.full_a[as], (BS / 64) * 128 * P.a_rows);
#pragma unroll
        for (int kc = 0; kc < BS / 64; ++kc)
          tma_load_2d(astage + as * C::kAStage + kc * (kTM * 128), &P.txp, &bars.full_a[as],
                      B * BS + kc * 64, m0);
        ++issued;
        if (MODE == kDynamic && cs > 1 && w == nbc - 1) {
          cluster_arrive_relaxed();
          arrived1 = true;
        }
        // the parts of the next block: they wait only for the MMAs of blocks
        // whose A tiles are already out
        while (ok && ur < min(U, 3 * (w + 2))) ok = issue_r(ur++);
      }
      // never leave with copies in flight
      for (int u = max(0, ur - C::kRS); u < ur; ++u)
        mbar_wait(&bars.full_r[u % C::kRS], (u / C::kRS) & 1, err);
      for (int w = max(0, issued - C::kAS); w < issued; ++w)
        mbar_wait(&bars.full_a[w % C::kAS], (w / C::kAS) & 1, err);
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------- R_B parts
    if (lane == 0) {
      for (int w = 0; w < W; ++w) {
        const int B = B0 + w % nbc;
        for (int sp = 0; sp < 3; ++sp) {
          const int u = 3 * w + sp, rr = u % C::kRS;
          if (!mbar_wait(&bars.empty_r[rr], ((u / C::kRS) & 1) ^ 1u, err)) break;
          mbar_arrive_expect_tx(&bars.full_r[rr], C::kRStage);
          bulk_copy_g2s(rstage + rr * C::kRStage,
                        P.rot_tc + (static_cast<size_t>(B) * 3 + sp) * BS * BS, C::kRStage,
                        &bars.full_r[rr]);
        }
        if (MODE == kDynamic && cs > 1 && w == nbc - 1) {
          cluster_arrive_relaxed();
          arrived1 = true;
        }
      }
      // never leave with copies in flight
      const int U = 3 * W;
      for (int u = U - C::kRS < 0 ? 0 : U - C::kRS; u < U; ++u)
        mbar_wait(&bars.full_r[u % C::kRS], (u / C::kRS) & 1, err);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTM, BS);
      const uint32_t a_base = smem_u32(astage), r_base = smem_u32(rstage);
      for (int w = 0; w < W; ++w) {
        const int as = w % C::kAS, ab = w & 1;
        if (!mbar_wait(&bars.full_a[as], (w / C::kAS) & 1, err)) break;
        if (!mbar_wait(&bars.acc_empty[ab], ((w >> 1) & 1) ^ 1u, err)) break;
        // when the ring holds whole blocks, the block's three R_B parts are
        // all waited for before the first MMA (a wait issued right behind
        // MMAs costs far more than one ahead); otherwise part by part, so
        // that the MMAs of the first parts free ring slots for the next
        constexpr bool kWhole = C::kRS % 3 == 0;
        bool okr = true;
        for (int sp = 0; kWhole && sp < 3 && okr; ++sp)
          okr = mbar_wait(&bars.full_r[(3 * w + sp) % C::kRS], ((3 * w + sp) / C::kRS) & 1, err);
        if (!okr) break;
        if (kWhole) tc_fence_after();
        for (int sp = 0; sp < 3 && okr; ++sp) {
          const int rr = (3 * w + sp) % C::kRS;
          if (!kWhole) {
            okr = mbar_wait(&bars.full_r[rr], ((3 * w + sp) / C::kRS) & 1, err);
            if (!okr) break;
            tc_fence_after();
          }
#pragma unroll
          for (int k = 0; k < BS / 16; ++k) {
            const int kc = k >> 2, kk = k & 3;
            const uint64_t ad = smem_desc_kmajor_sw128(a_base + as * C::kAStage + kc * (kTM * 128) + kk * 32);
            const uint64_t bd = smem_desc_kmajor_sw128(r_base + rr * C::kRStage + kc * (BS * 128) + kk * 32);
            umma_bf16(tmem + ab * BS, ad, bd, idesc, (sp | k) != 0 ? 1u : 0u);
          }
          if (!kWhole) umma_commit(&bars.empty_r[rr]);
        }
        if (!okr) break;
        if (kWhole)
          for (int sp = 0; sp < 3; ++sp) umma_commit(&bars.empty_r[(3 * w + sp) % C::kRS]);
        umma_commit(&bars.empty_a[as]);
        umma_commit(&bars.acc_full[ab]);
        if (MODE == kDynamic && cs > 1 && w == nbc - 1) {
          cluster_arrive_relaxed();
          arrived1 = true;
        }
      }
    }
  } else if (!epi) {
    // ----------------------------------------------- gather (no TMA route)
    const int t = tid - 64;                    // token row of the tile
    pdl_wait();
    const bool valid = t < ntok;
    const __nv_bfloat16* xrow = x + static_cast<size_t>(m0 + (valid ? t : 0)) * ldx;
    for (int w = 0; w < W; ++w) {
      const int B = B0 + w % nbc, as = w % C::kAS;
      const int32_t* pB = P.perm + static_cast<size_t>(B) * BS;
      uint32_t v[BS / 2];
#pragma unroll
      for (int i = 0; i < BS; i += 2) {
        uint32_t lo = 0, hi = 0;
        if (valid) {
          const int p0 = __ldg(pB + i), p1 = __ldg(pB + i + 1);
          lo = __ldg(reinterpret_cast<const unsigned short*>(xrow) + (static_cast<unsigned>(p0) < static_cast<unsigned>(K) ? p0 : 0));
          hi = __ldg(reinterpret_cast<const unsigned short*>(xrow) + (static_cast<unsigned>(p1) < static_cast<unsigned>(K) ? p1 : 0));
        }
        v[i / 2] = lo | (hi << 16);
      }
      if (!mbar_wait(&bars.empty_a[as], ((w / C::kAS) & 1) ^ 1u, err)) break;
      uint8_t* at = astage + as * C::kAStage;
#pragma unroll
      for (int c8 = 0; c8 < BS / 8; ++c8) {
        const int kc = c8 >> 3, c = c8 & 7;
        *reinterpret_cast<uint4*>(at + kc * (kTM * 128) + t * 128 + ((c ^ (t & 7)) << 4)) =
            make_uint4(v[4 * c8], v[4 * c8 + 1], v[4 * c8 + 2], v[4 * c8 + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars.full_a[as]);
      if (MODE == kDynamic && cs > 1 && w == nbc - 1) {
        cluster_arrive_relaxed();
        arrived1 = true;
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int t = q4 * 32 + lane;              // token row = TMEM lane
    constexpr int kCols = BS / kHalves;        // accumulator columns of this thread
    const int cbeg = ((warp - kFirstEpi) >> 2) * kCols;
    const bool valid = t < ntok;
    pdl_wait();
    pdl_launch_dependents();
    float s = 0.f;
    if (MODE == kTable) s = table_scale(P.table, P.T, P.Lcount, P.step_dev, P.step_host, P.layer, err);
    float amax = 0.f;
    bool reduced = false;
    // row maximum over both column halves and every CTA of the cluster that
    // shares these tokens (once per thread, also when this CTA holds no block
    // or gave up early); maxima of non-negative floats order as their bits
    auto reduce_rows = [&]() {
      if (kHalves > 1 || cs > 1) atomicMax(&amax_s[t], __float_as_uint(amax));
      if (kHalves > 1 && cs == 1) {
        named_barrier(1, 32 * kEpiWarps);
        amax = __uint_as_float(amax_s[t]);
      }
      if (cs > 1) {
        asm volatile("barrier.cluster.arrive.release;" ::: "memory");
        asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
        unsigned int mx = 0u;
        const uint32_t a = smem_u32(&amax_s[t]);
        for (int r2 = 0; r2 < cs; ++r2) {
          uint32_t v;
          asm volatile("ld.shared::cluster.u32 %0, [%1];"
                       : "=r"(v)
                       : "r"(map_shared_rank(a, static_cast<uint32_t>(r2)))
                       : "memory");
          mx = max(mx, v);
        }
        cluster_arrive_relaxed();          // phase 2: done reading peers
        amax = __uint_as_float(mx);
      }
      if (phase == 1 && valid && cbeg == 0)
        P.amax[static_cast<size_t>(group) * M + m0 + t] = __float_as_uint(amax);
      s = __fdiv_rn(amax, 7.0f);
      reduced = true;
    };
    if (MODE == kDynamic && phase == 2) {
      // the row maximum over the maxima of every CTA of the first launch that
      // held these tokens (written before it completed, which pdl_wait above
      // waited for)
      unsigned int mx = 0u;
      if (valid)
        for (int g = 0; g < P.ngroups; ++g)
          mx = max(mx, __ldcg(P.amax + static_cast<size_t>(g) * M + m0 + t));
      amax = __uint_as_float(mx);
      s = __fdiv_rn(amax, 7.0f);
      reduced = true;
    }
    // 32-byte aligned outputs take 32-byte stores (each row's offsets are
    // multiples of 32 bytes: K is a multiple of 64)
    const bool xq32 = (reinterpret_cast<uintptr_t>(P.xq) & 31u) == 0;
    const bool xq8_32 = (reinterpret_cast<uintptr_t>(P.xq8) & 31u) == 0;
    uint4 keep = make_uint4(0u, 0u, 0u, 0u);
    for (int w = 0; w < W; ++w) {
      const int ab = w & 1, pass = phase == 0 ? w / nbc : phase - 1, B = B0 + w % nbc;
      // one outcome per warp, and a converged warp for the warp-wide loads
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.acc_full[ab], (w >> 1) & 1, err))) break;
      tc_fence_after();
      const float a15 = quant_recip15(s);
#pragma unroll 1
      for (int c0 = cbeg; c0 < cbeg + kCols; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q4 * 32) << 16) + ab * BS + c0, r);
        tmem_ld_wait();
        if (MODE == kRotateOnly) {
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(P.xr_out + static_cast<size_t>(m0 + t) * K + B * BS + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                   __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
          }
        } else if (MODE == kDynamic && pass == 0) {
#pragma unroll
          for (int c = 0; c < 32; ++c) amax = fmaxf(amax, fabsf(__uint_as_float(r[c])));
        } else {
          // two halves of 16 codes: half the registers of one pass
          uint32_t wv[4];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float f[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) f[c] = __uint_as_float(r[16 * hh + c]);
            uint32_t w2[2];
            quant_pack<16>(f, s, a15, w2);
            wv[2 * hh] = w2[0];
            wv[2 * hh + 1] = w2[1];
          }
          if (valid) {
            // full 32-byte sectors where the buffers allow (one request per
            // sector instead of two): the codes of two 32-column chunks go
            // out together, the image of a chunk in one store
            uint8_t* dq = P.xq + static_cast<size_t>(m0 + t) * (K / 2) + (B * BS + c0) / 2;
            const uint4 cw = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            if (kCols % 64 == 0 && xq32) {
              if (((c0 - cbeg) & 32) == 0)
                keep = cw;                          // first chunk of a pair (32-byte aligned)
              else
                st_global_v8(dq - 16, keep, cw);
            } else {
              *reinterpret_cast<uint4*>(dq) = cw;
            }
            if (P.xq8 != nullptr) {
              // the GEMM's int8 image of these 32 codes: 16*q, even codes
              // first, then odd codes
              int8_t* d8 = P.xq8 + static_cast<size_t>(m0 + t) * K + B * BS + c0;
              const uint4 lo = make_uint4((wv[0] << 4) & 0xF0F0F0F0u, (wv[1] << 4) & 0xF0F0F0F0u,
                                          (wv[2] << 4) & 0xF0F0F0F0u, (wv[3] << 4) & 0xF0F0F0F0u);
              const uint4 hi = make_uint4(wv[0] & 0xF0F0F0F0u, wv[1] & 0xF0F0F0F0u, wv[2] & 0xF0F0F0F0u,
                                          wv[3] & 0xF0F0F0F0u);
              if (xq8_32) {
                st_global_v8(d8, lo, hi);
              } else {
                reinterpret_cast<uint4*>(d8)[0] = lo;
                reinterpret_cast<uint4*>(d8)[1] = hi;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[ab]);
      if (MODE == kDynamic && phase < 2 && w == nbc - 1) reduce_rows();
    }
    if (MODE == kDynamic && !reduced) reduce_rows();
    if (MODE != kRotateOnly && phase != 1 && group == 0 && valid && cbeg == 0) P.s_x[m0 + t] = s;
  }

  if (MODE == kDynamic && cs > 1) {
    if (!epi) {
      if (!arrived1) cluster_arrive_relaxed();   // idle lanes, early exits
      cluster_wait();                            // phase 1
      cluster_arrive_relaxed();                  // phase 2
    }
    cluster_wait();                              // phase 2: peers done with our smem
  }
  cta_sync();
  if (warp == 1) {
    __syncwarp();                  // lane 0 comes from the MMA loop
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Permuted copy of bf16 rows: out[m][j] = x[m][perm[j]].  One CTA per run of
// `rpc` consecutive rows of one problem, as a pipeline over a ring of row
// buffers in shared memory:
//   warp 8      bulk-copies whole rows (16-byte aligned, K * 2 bytes) into
//               the ring, one mbarrier per slot
//   warps 0-7   in groups of `gw` warps, each group one row at a time (rows
//               g, g + groups, ...): every thread takes its runs of 8 output
//               positions, gathers them from the staged row and writes them
//               with one 16-byte store (coalesced); the permutation entries
//               of its runs stay in registers for all rows
// so the loads of later rows are in flight while earlier rows are scattered,
// and short rows are scattered several at a time.  Slot st always serves
// group st % groups (the slot count is a multiple of the group count), so a
// group never waits on a slot phase that another group has yet to consume.
struct PermJob {
  const __nv_bfloat16* x;
  const int32_t* perm;
  __nv_bfloat16* out;
  int ldx, M, K;
  int rpc;                          // rows per CTA
  int stages;                       // row slots of K * 2 bytes in the ring
  int gw;                           // warps per row group: 1, 2, 4 or 8
};
constexpr int kPermMaxStages = 32;
constexpr int kPermWorkers = 256;
struct PermBatch {
  int n;
  int cta_start[kMaxBatch + 1];
  PermJob j[kMaxBatch];
};

// kPC: runs of 8 positions per worker thread (K <= 2048 * kPC)
template <int kPC>
__global__ void __launch_bounds__(kPermWorkers + 32)
    permute_rows_kernel(const __grid_constant__ PermBatch batch, unsigned int* err) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kPermMaxStages], empty[kPermMaxStages];
  int ji = 0;
  while (ji + 1 < batch.n && static_cast<int>(blockIdx.x) >= batch.cta_start[ji + 1]) ++ji;
  const PermJob& J = batch.j[ji];
  const int r0 = (static_cast<int>(blockIdx.x) - batch.cta_start[ji]) * J.rpc;
  const int nr = min(J.rpc, J.M - r0);
  const int K = J.K, kc = K / 8, S = J.stages;
  const int row_bytes = K * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gthr = 32 * J.gw, ng = kPermWorkers / gthr;   // threads per group, groups
  const int grp = tid / gthr, gt = tid - grp * gthr;      // this worker's group, index in it
  // the permutation does not depend on the previous kernel: read before
  // waiting for it
  int p[kPC][8];
#pragma unroll
  for (int c = 0; c < kPC; ++c) {
    const int i = gt + gthr * c;
    int4 a = make_int4(0, 0, 0, 0), b = make_int4(0, 0, 0, 0);
    if (tid < kPermWorkers && i < kc) {
      a = __ldg(reinterpret_cast<const int4*>(J.perm) + 2 * i);
      b = __ldg(reinterpret_cast<const int4*>(J.perm) + 2 * i + 1);
    }
    const int q[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int u = 0; u < 8; ++u) p[c][u] = static_cast<unsigned>(q[u]) < static_cast<unsigned>(K) ? q[u] : 0;
  }
  if (tid == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], gthr);
    }
    fence_mbar_init();
  }
  cta_sync();
  pdl_wait();
  pdl_launch_dependents();
  if (warp == kPermWorkers / 32) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int r = 0; r < nr; ++r) {
        const int st = r % S;
        if (!mbar_wait(&empty[st], ((r / S) & 1) ^ 1u, err)) break;
        mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(K) * 2u);
        bulk_copy_g2s(smem + static_cast<size_t>(st) * row_bytes,
                      J.x + static_cast<size_t>(r0 + r) * J.ldx, static_cast<uint32_t>(K) * 2u, &full[st]);
        ++issued;
      }
      // never leave with copies in flight
      for (int r = max(0, issued - S); r < issued; ++r) mbar_wait(&full[r % S], (r / S) & 1, err);
    }
  } else {
    // ------------------------------------------------------------- workers
    for (int r = grp; r < nr; r += ng) {
      const int st = r % S;
      if (!mbar_wait(&full[st], (r / S) & 1, err)) break;
      const unsigned short* sr =
          reinterpret_cast<const unsigned short*>(smem + static_cast<size_t>(st) * row_bytes);
      uint4* orow = reinterpret_cast<uint4*>(J.out + static_cast<size_t>(r0 + r) * K);
#pragma unroll
      for (int c = 0; c < kPC; ++c) {
        const int i = gt + gthr * c;
        if (i < kc) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            w[q] = static_cast<uint32_t>(sr[p[c][2 * q]]) | (static_cast<uint32_t>(sr[p[c][2 * q + 1]]) << 16);
          orow[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      mbar_arrive(&empty[st]);
    }
  }
}

// The GEMM's int8 image of packed codes, for the routes that write only the
// packed form: every 16 packed bytes (32 codes) become 32 image bytes, 16*q
// of the even codes, then of the odd codes.
struct ExpandJob {
  const uint8_t* xq;
  int8_t* xq8;
};
struct ExpandBatch {
  int n;
  long long start[kMaxBatch + 1];   // prefix sums of 16-byte packed chunks
  ExpandJob j[kMaxBatch];
};

__global__ void __launch_bounds__(256) expand_codes_kernel(const __grid_constant__ ExpandBatch b) {
  pdl_wait();
  pdl_launch_dependents();
  const long long total = b.start[b.n];
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    int ji = 0;
    while (ji + 1 < b.n && u >= b.start[ji + 1]) ++ji;
    const long long local = u - b.start[ji];
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(b.j[ji].xq) + local);
    uint4* d = reinterpret_cast<uint4*>(b.j[ji].xq8) + 2 * local;
    d[0] = make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u, (w.z << 4) & 0xF0F0F0F0u,
                      (w.w << 4) & 0xF0F0F0F0u);
    d[1] = make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
  }
}

cudaError_t launch_expand(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  std::vector<const ActArgs*> w;
  for (const ActArgs* a : v)
    if (a->xq8 != nullptr && a->xq != nullptr && a->M > 0) w.push_back(a);
  for (size_t i0 = 0; i0 < w.size(); i0 += kMaxBatch) {
    const int n = static_cast<int>(std::min<size_t>(kMaxBatch, w.size() - i0));
    ExpandBatch b;
    std::memset(&b, 0, sizeof(b));
    b.n = n;
    long long chunks = 0;
    for (int i = 0; i < n; ++i) {
      b.j[i].xq = w[i0 + i]->xq;
      b.j[i].xq8 = w[i0 + i]->xq8;
      b.start[i] = chunks;
      chunks += static_cast<long long>(w[i0 + i]->M) * (w[i0 + i]->K / 32);
    }
    b.start[n] = chunks;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<long long>((chunks + 255) / 256, 148 * 8)), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, expand_codes_kernel, b);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

// Quantise fp32 rows (already rotated): one CTA per row, the rows of up to
// kMaxBatch independent sets in one launch.
struct QuantJob {
  const float* xr;
  const float* table;
  const int32_t* step_dev;
  uint8_t* q_out;
  float* s_out;
  int K, qmin, qmax, dynamic, T, Lcount, step_host, layer, bits;
};
struct QuantBatch {
  int n;
  int row_start[kMaxBatch + 1];   // first CTA of each set
  QuantJob j[kMaxBatch];
};

__global__ void __launch_bounds__(kThreads)
    quant_rows_kernel(const __grid_constant__ QuantBatch batch, unsigned int* err) {
  __shared__ float red[kWarps];
  __shared__ float s_sh;
  int ji = 0;
  while (ji + 1 < batch.n && static_cast<int>(blockIdx.x) >= batch.row_start[ji + 1]) ++ji;
  const QuantJob& J = batch.j[ji];
  const float* __restrict__ xr = J.xr;
  uint8_t* __restrict__ q_out = J.q_out;
  float* __restrict__ s_out = J.s_out;
  const int K = J.K, qmin = J.qmin, qmax = J.qmax, bits = J.bits;
  const int row = static_cast<int>(blockIdx.x) - batch.row_start[ji], tid = threadIdx.x;
  const float* src = xr + static_cast<size_t>(row) * K;
  if (J.dynamic) {
    float mx = 0.f;
    for (int k = tid; k < K; k += kThreads) mx = fmaxf(mx, fabsf(src[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    cta_sync();
    if (tid == 0) {
      float m = 0.f;
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w]);
      s_sh = __fdiv_rn(m, static_cast<float>(qmax));
    }
  } else if (tid == 0) {
    s_sh = table_scale(J.table, J.T, J.Lcount, J.step_dev, J.step_host, J.layer, err);
  }
  cta_sync();
  const float s = s_sh;
  if (bits == 8) {
    // one int8 code per byte, decided by the IEEE fp32 division itself
    int8_t* dst8 = reinterpret_cast<int8_t*>(q_out) + static_cast<size_t>(row) * K;
    for (int j = tid; j < K; j += kThreads)
      dst8[j] = static_cast<int8_t>(quant_code(src[j], s, qmin, qmax));
    if (tid == 0) s_out[row] = s;
    return;
  }
  uint8_t* dst = q_out + static_cast<size_t>(row) * (K / 2);
  if (qmin == -8 && qmax == 7 && K % 8 == 0) {
    // activations: the epilogue quantiser of the rotation kernels, 8 values
    // (one 32-bit word of codes) per thread
    const float a15 = quant_recip15(s);
    for (int j = tid; j < K / 8; j += kThreads) {
      float f[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) f[u] = src[8 * j + u];
      uint32_t wd[1];
      quant_pack<8>(f, s, a15, wd);
      *reinterpret_cast<uint32_t*>(dst + 4 * j) = wd[0];
    }
    if (tid == 0) s_out[row] = s;
    return;
  }
  const float rs = quant_recip(s);
  for (int j = tid; j < K / 2; j += kThreads) {
    const int q0 = quant_code_fast(src[2 * j], s, rs, qmin, qmax);
    const int q1 = quant_code_fast(src[2 * j + 1], s, rs, qmin, qmax);
    dst[j] = static_cast<uint8_t>((q0 & 15) | ((q1 & 15) << 4));
  }
  if (tid == 0) s_out[row] = s;
}

// Grid of one problem: token tiles gx, CTAs per token tile (block groups, or
// the cluster size in DYNAMIC mode) and rotation blocks per CTA.
template <int BS, int TT, int MODE>
void problem_grid(int M, int K, int* gx, int* per_tile, int* bpc, int min_bpc = 1) {
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
    *bpc = std::min(nb, std::max((nb + g - 1) / g, min_bpc));
    *per_tile = (nb + *bpc - 1) / *bpc;
  }
}

// Launches up to kMaxBatch problems that share (BS, TT, Tin, MODE) and, in
// DYNAMIC mode, the cluster size.
template <int BS, int TT, typename Tin, int MODE>
cudaError_t launch_group(const ActArgs* const* as, int n, cudaStream_t stream, int min_bpc = 1) {
  ActBatch batch;
  std::memset(&batch, 0, sizeof(batch));
  batch.n = n;
  int ctas = 0, cs = 1, bpc_max = 1;
  for (int i = 0; i < n; ++i) {
    const ActArgs& a = *as[i];
    int gx, per_tile, bpc;
    problem_grid<BS, TT, MODE>(a.M, a.K, &gx, &per_tile, &bpc, min_bpc);
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
  static std::atomic<unsigned long long> attr_done{0};
  {
    cudaError_t e = once_per_device(attr_done, [&]() {
      cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
      if (r == cudaSuccess && MODE == kDynamic)
        r = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      return r;
    });
    if (e != cudaSuccess) return e;
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
    // Each problem alone would be cut into ~2 CTAs per SM; a batch of them
    // shares the GPU, so the blocks per CTA are raised until the launch fits
    // in one wave (4 resident CTAs per SM), rather than leave a second wave
    // of a few CTAs.
    for (size_t i0 = 0; i0 < v.size(); i0 += kMaxBatch) {
      const int n = static_cast<int>(std::min<size_t>(kMaxBatch, v.size() - i0));
      int min_bpc = 1;
      for (;;) {
        int ctas = 0;
        for (int i = 0; i < n; ++i) {
          int gx, per_tile, bpc;
          problem_grid<BS, TT, MODE>(v[i0 + i]->M, v[i0 + i]->K, &gx, &per_tile, &bpc, min_bpc);
          ctas += gx * per_tile;
        }
        if (ctas <= 4 * 148 || min_bpc >= 64) break;
        min_bpc *= 2;
      }
      cudaError_t e = launch_group<BS, TT, Tin, MODE>(v.data() + i0, n, stream, min_bpc);
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

// QVLA_ROTATE_PATH=fma: every problem on the R_SVD + Walsh-Hadamard
// CUDA-core kernel (no tensor cores, no composite kernel), for tests.
bool rsvd_path_forced() {
  const char* p = std::getenv("QVLA_ROTATE_PATH");
  return p && std::strcmp(p, "fma") == 0;
}

// Composite-path launches: every (token tile, block) pair of a launch gets a
// CTA while they fit eight per SM; beyond that each CTA walks several blocks.
template <typename Tin, int MODE>
cudaError_t launch_comp(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  const long long slots = 8LL * 148;
  for (size_t i0 = 0; i0 < v.size(); i0 += kMaxBatch) {
    const int n = static_cast<int>(std::min<size_t>(kMaxBatch, v.size() - i0));
    long long pairs = 0;
    for (int i = 0; i < n; ++i)
      pairs += static_cast<long long>((v[i0 + i]->M + kCTT - 1) / kCTT) * (v[i0 + i]->K / kCBS);
    const int bpc = static_cast<int>(std::max<long long>(1, (pairs + slots - 1) / slots));
    ActBatch batch;
    std::memset(&batch, 0, sizeof(batch));
    batch.n = n;
    int ctas = 0;
    for (int i = 0; i < n; ++i) {
      const ActArgs& a = *v[i0 + i];
      ActProblem& P = batch.p[i];
      P.x = a.x;
      P.perm = a.perm;
      P.rot = a.rot;
      P.rot_tc = a.rot_tc;
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
      P.gx = (a.M + kCTT - 1) / kCTT;
      P.bpc = std::min(bpc, a.K / kCBS);
      batch.cta_start[i] = ctas;
      ctas += P.gx * ((a.K / kCBS + P.bpc - 1) / P.bpc);
    }
    batch.cta_start[n] = ctas;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas, 1, 1);
    cfg.blockDim = dim3(kCThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, rotq_comp_kernel<Tin, MODE>, batch, device_error_word());
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <int BS, typename Tin, int MODE>
cudaError_t launch_bs(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  std::vector<const ActArgs*> comp, t16, t32;
  for (const ActArgs* a : v) {
    if (BS == kCBS && MODE != kDynamic && a->rot_tc != nullptr && !rsvd_path_forced())
      comp.push_back(a);
    else
      (token_tile_for(a->M, a->K, BS, MODE) == 16 ? t16 : t32).push_back(a);
  }
  cudaError_t e = cudaSuccess;
  if (!comp.empty()) e = launch_comp<Tin, MODE>(comp, stream);
  if (e == cudaSuccess && !t16.empty()) e = launch_cfg_batches<BS, 16, Tin, MODE>(t16, stream);
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

// ---------------------------------------------------------------- TC host
template <int BS, bool kLat = false>
int tc_ctas_per_sm() {
  return kLat ? 3 : TcCfg<BS>::kSmem <= 110 * 1024 ? 2 : 1;
}

template <int BS>
int tc_cluster(int M, int K) {
  const int gx = (M + kTM - 1) / kTM, nb = K / BS;
  const int slots = 148 * tc_ctas_per_sm<BS>();
  int cs = 1;
  while (cs < 16 && 2 * cs <= nb && gx * cs < slots) cs *= 2;
  return cs;
}

// Rows of the permuted-x box: the batch's token count rounded up to 16, at
// most one 128-token tile.
int xperm_box_rows(int M) { return std::min(kTM, (M + 15) / 16 * 16); }

bool make_xperm_map(CUtensorMap* map, void* ptr, int M, int K) {
  static const EncodeTiledFnR enc = []() -> EncodeTiledFnR {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFnR>(p);
  }();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(xperm_box_rows(M))};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Permuted copies x_perm = x[:, perm] of the problems that have scratch.
// Each CTA's ring is about 48 KB (128 KB for the longest rows, whose variant
// holds the permutation of 16 runs per thread in registers and so runs one
// CTA per SM), cut into as many slots as it holds of the CTA's own rows (2 to
// 32); the elements of a launch are spread evenly over the CTAs (fewer rows
// per CTA where the rows are longer).
template <int kPC>
int permute_ring_bytes() { return kPC >= 16 ? 128 * 1024 : 48 * 1024; }

// CTAs per SM the register file allows (shared memory is counted by the caller).
template <int kPC>
int permute_reg_occupancy() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  int c = cache[dev].load(std::memory_order_relaxed);
  if (c > 0) return c;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c, permute_rows_kernel<kPC>, kPermWorkers + 32, 0) !=
          cudaSuccess || c <= 0) {
    cudaGetLastError();
    c = 1;
  }
  cache[dev].store(c, std::memory_order_relaxed);
  return c;
}

template <int kPC>
cudaError_t launch_permute_kernel(PermBatch& b, const ActArgs* const* as, int kmax,
                                  cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = once_per_device(attr_done, []() {
    return cudaFuncSetAttribute(permute_rows_kernel<kPC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                2 * QVLA_MAX_K * 2);
  });
  if (e != cudaSuccess) return e;
  // one ring of shared memory per CTA, as many row slots as it holds for the
  // CTA's own rows (so short rows keep more of them in flight)
  const int smem = std::max(permute_ring_bytes<kPC>(), 2 * kmax * 2);
  for (int i = 0; i < b.n; ++i) {
    // rows scattered at a time: groups of the fewest warps whose threads hold
    // the row's runs of 8 (kPC each), while the ring keeps two slots per group
    const int K = as[i]->K, slots = std::min(kPermMaxStages, smem / (K * 2));
    int gw = 1;
    while (gw < kPermWorkers / 32 && (K / 8 > 32 * gw * kPC || slots < 2 * (kPermWorkers / 32 / gw))) gw *= 2;
    const int ng = kPermWorkers / 32 / gw;
    b.j[i].gw = gw;
    b.j[i].stages = slots / ng * ng;               // a multiple of the group count
  }
  // the elements spread over one wave of resident CTAs; the longest rows
  // (one CTA per SM) take three CTAs per SM in waves, measured faster than
  // one long CTA per SM
  const int occ = kPC >= 16 ? 3
                            : std::max(1, std::min(permute_reg_occupancy<kPC>(), 227 * 1024 / (smem + 2048)));
  long long elems = 0;
  for (int i = 0; i < b.n; ++i) elems += static_cast<long long>(as[i]->M) * as[i]->K;
  const long long slots = 148LL * occ;
  const long long per_cta = (elems + slots - 1) / slots;
  int ctas = 0;
  for (int i = 0; i < b.n; ++i) {
    b.j[i].rpc = static_cast<int>(std::max<long long>(1, (per_cta + as[i]->K - 1) / as[i]->K));
    b.cta_start[i] = ctas;
    ctas += (as[i]->M + b.j[i].rpc - 1) / b.j[i].rpc;
  }
  b.cta_start[b.n] = ctas;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas, 1, 1);
  cfg.blockDim = dim3(kPermWorkers + 32, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, permute_rows_kernel<kPC>, b, device_error_word());
}

cudaError_t launch_permute(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  for (size_t i0 = 0; i0 < v.size(); i0 += kMaxBatch) {
    const int n = static_cast<int>(std::min<size_t>(kMaxBatch, v.size() - i0));
    PermBatch b;
    std::memset(&b, 0, sizeof(b));
    b.n = n;
    int kmax = 0;
    for (int i = 0; i < n; ++i) {
      const ActArgs& a = *v[i0 + i];
      kmax = std::max(kmax, a.K);
      b.j[i].x = static_cast<const __nv_bfloat16*>(a.x);
      b.j[i].perm = a.perm;
      b.j[i].out = static_cast<__nv_bfloat16*>(a.ws);
      b.j[i].ldx = a.ldx;
      b.j[i].M = a.M;
      b.j[i].K = a.K;
    }
    const int runs = (kmax / 8 + kPermWorkers - 1) / kPermWorkers;   // runs of 8 per thread
    const ActArgs* const* as = v.data() + i0;
    cudaError_t e = runs <= 1   ? launch_permute_kernel<1>(b, as, kmax, stream)
                    : runs <= 4 ? launch_permute_kernel<4>(b, as, kmax, stream)
                                : launch_permute_kernel<16>(b, as, kmax, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

// One launch of up to kMaxBatch problems sharing (BS, MODE) and, in DYNAMIC
// mode, the cluster size `cs`; TABLE / rotate-only and the two DYNAMIC
// phases (`phase` 1, 2: see ActBatch) take `G` blocks per CTA.
template <int BS, int MODE, bool kTmaA, bool kLat = false>
cudaError_t launch_tc_group(const ActArgs* const* as, int n, int G, int cs, cudaStream_t stream,
                            int phase = 0) {
  using C = TcCfg<BS, kLat>;
  ActBatch batch;
  std::memset(&batch, 0, sizeof(batch));
  batch.n = n;
  batch.phase = phase;
  int ctas = 0;
  for (int i = 0; i < n; ++i) {
    const ActArgs& a = *as[i];
    ActProblem& P = batch.p[i];
    if (kTmaA && !make_xperm_map(&P.txp, a.ws, a.M, a.K)) return cudaErrorInvalidValue;
    P.x = a.x;
    P.perm = a.perm;
    P.rot = a.rot;
    P.rot_tc = a.rot_tc;
    P.table = a.table;
    P.step_dev = a.step_dev;
    P.xq = a.xq;
    P.xq8 = a.xq8;
    P.s_x = a.s_x;
    P.xr_out = a.xr_out;
    P.M = a.M;
    P.ldx = a.ldx;
    P.K = a.K;
    P.T = a.T;
    P.Lcount = a.Lcount;
    P.step_host = a.step_host;
    P.layer = a.layer;
    const int nb = a.K / BS;
    P.gx = (a.M + kTM - 1) / kTM;
    P.a_rows = xperm_box_rows(a.M);
    batch.cta_start[i] = ctas;
    if (MODE == kDynamic && phase == 0) {
      P.bpc = (nb + cs - 1) / cs;
      ctas += P.gx;
    } else {
      P.bpc = std::min(G, nb);
      ctas += P.gx * ((nb + P.bpc - 1) / P.bpc);
      if (MODE == kDynamic) {
        // the maxima follow the permuted copy in the scratch
        P.amax = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(a.ws) +
                                                 static_cast<size_t>(a.M) * a.K * 2);
        P.ngroups = (nb + P.bpc - 1) / P.bpc;
      }
    }
  }
  batch.cta_start[n] = ctas;
  auto kern = rotq_tc_kernel<BS, MODE, kTmaA, kLat>;
  static std::atomic<unsigned long long> attr_done{0};
  {
    cudaError_t e = once_per_device(attr_done, [&]() {
      cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      // the grid is sized for tc_ctas_per_sm() CTAs per SM: ask for the
      // shared-memory carveout that holds them
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
      return r;
    });
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas, MODE == kDynamic && phase == 0 ? cs : 1, 1);
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
  if (MODE == kDynamic && phase == 0 && cs > 1) {
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

// DYNAMIC launch costs, in passes of one CTA over one rotation block (a
// launch adds one): the one-launch route with a cluster along the blocks,
// and the two-launch route (maxima, then quantisation) with `G` blocks per
// CTA and no cluster.  Both assume the CTAs that fit one wave run together.
template <int BS>
long long cluster_route_cost(const std::vector<const ActArgs*>& v, long long slots) {
  long long cost = 0;
  for (int cs = 1; cs <= 16; cs *= 2) {
    std::vector<const ActArgs*> g;
    for (const ActArgs* a : v)
      if (tc_cluster<BS>(a->M, a->K) == cs) g.push_back(a);
    for (size_t i0 = 0; i0 < g.size(); i0 += kMaxBatch) {
      const size_t n = std::min<size_t>(kMaxBatch, g.size() - i0);
      long long tiles = 0, per = 0;
      for (size_t i = 0; i < n; ++i) tiles += (g[i0 + i]->M + kTM - 1) / kTM;
      int c = cs;
      while (c > 1 && tiles * c > slots) c /= 2;
      for (size_t i = 0; i < n; ++i) per = std::max<long long>(per, (g[i0 + i]->K / BS + c - 1) / c);
      cost += 2 * per * ((tiles * c + slots - 1) / slots) + 1;
    }
  }
  return cost;
}

template <int BS>
int split_route_blocks(const ActArgs* const* as, int n, long long slots, long long* cost) {
  int nbmax = 1;
  for (int i = 0; i < n; ++i) nbmax = std::max(nbmax, as[i]->K / BS);
  long long best = -1;
  int bestG = 1;
  for (int G = 1; G <= nbmax; ++G) {
    long long ctas = 0;
    for (int i = 0; i < n; ++i) {
      const int nb = as[i]->K / BS, g = std::min(G, nb);
      ctas += static_cast<long long>((as[i]->M + kTM - 1) / kTM) * ((nb + g - 1) / g);
    }
    const long long c = (ctas + slots - 1) / slots * G;
    if (best < 0 || c <= best) {           // ties: fewer, longer CTAs
      best = c;
      bestG = G;
    }
  }
  *cost = 2 * (best + 1);
  return bestG;
}

// scratch for the two-launch DYNAMIC route: the permuted copy, then the row
// maxima of up to K / BS CTAs per token
template <int BS>
bool has_amax_scratch(const ActArgs* a) {
  return a->ws_bytes >= static_cast<size_t>(a->M) * a->K * 2 + static_cast<size_t>(a->M) * (a->K / BS) * 4;
}

template <int BS, int MODE, bool kTmaA>
cudaError_t launch_tc_mode(const std::vector<const ActArgs*>& v, cudaStream_t stream) {
  if (v.empty()) return cudaSuccess;
  if (MODE == kDynamic) {
    const long long slots = 148LL * tc_ctas_per_sm<BS>();
    if (kTmaA) {
      // two launches per batch when every problem has room for the maxima and
      // that is shorter: the blocks of wide and narrow linears then spread
      // evenly over the SMs, where one cluster size per launch cannot
      bool room = true;
      for (const ActArgs* a : v) room = room && has_amax_scratch<BS>(a);
      if (room) {
        long long split = 0;
        std::vector<int> Gs;
        for (size_t i0 = 0; i0 < v.size(); i0 += kMaxBatch) {
          const int n = static_cast<int>(std::min<size_t>(kMaxBatch, v.size() - i0));
          long long c = 0;
          Gs.push_back(split_route_blocks<BS>(v.data() + i0, n, slots, &c));
          split += c;
        }
        if (split < cluster_route_cost<BS>(v, slots)) {
          for (size_t i0 = 0, k = 0; i0 < v.size(); i0 += kMaxBatch, ++k) {
            const int n = static_cast<int>(std::min<size_t>(kMaxBatch, v.size() - i0));
            cudaError_t e = launch_tc_group<BS, MODE, kTmaA>(v.data() + i0, n, Gs[k], 1, stream, 1);
            if (e == cudaSuccess) e = launch_tc_group<BS, MODE, kTmaA>(v.data() + i0, n, Gs[k], 1, stream, 2);
            if (e != cudaSuccess) return e;
          }
          return cudaSuccess;
        }
      }
    }
    // the cluster size each linear would take alone; a launch of several
    // halves it until all its clusters fit one wave (clusters of one CTA per
    // SM are only co-resident a GPC's worth at a time)
    for (int cs = 1; cs <= 16; cs *= 2) {
      std::vector<const ActArgs*> g;
      for (const ActArgs* a : v)
        if (tc_cluster<BS>(a->M, a->K) == cs) g.push_back(a);
      for (size_t i0 = 0; i0 < g.size(); i0 += kMaxBatch) {
        const int n = static_cast<int>(std::min<size_t>(kMaxBatch, g.size() - i0));
        long long tiles = 0;
        for (int i = 0; i < n; ++i) tiles += (g[i0 + i]->M + kTM - 1) / kTM;
        int c = cs;
        while (c > 1 && tiles * c > slots) c /= 2;
        cudaError_t e = launch_tc_group<BS, MODE, kTmaA>(g.data() + i0, n, 1, c, stream);
        if (e != cudaSuccess) return e;
      }
    }
    return cudaSuccess;
  }
  // blocks per CTA: spread each launch's (token tile, block) pairs over one
  // wave; a launch whose pairs fit one wave of the latency configuration
  // takes that (one block per CTA)
  const long long slots = 148LL * tc_ctas_per_sm<BS>();
  for (size_t i0 = 0; i0 < v.size(); i0 += kMaxBatch) {
    const int n = static_cast<int>(std::min<size_t>(kMaxBatch, v.size() - i0));
    long long pairs = 0;
    for (int i = 0; i < n; ++i)
      pairs += static_cast<long long>((v[i0 + i]->M + kTM - 1) / kTM) * (v[i0 + i]->K / BS);
    cudaError_t e;
    if constexpr (BS == 64 && MODE == kTable && kTmaA) {
      if (pairs <= 148LL * tc_ctas_per_sm<BS, true>()) {
        e = launch_tc_group<BS, MODE, kTmaA, true>(v.data() + i0, n, 1, 1, stream);
        if (e != cudaSuccess) return e;
        continue;
      }
    }
    const int G = static_cast<int>(std::max<long long>(1, (pairs + slots - 1) / slots));
    e = launch_tc_group<BS, MODE, kTmaA>(v.data() + i0, n, G, 1, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Token count from which the tensor-core rotation beats the CUDA-core ones:
// every M (50 tokens x 12 linears of a DiT step, table mode: 19.5 us through
// the permuted copy, 25.6 us gathering, against 27.7 us for the composite
// CUDA-core kernel and 31.7 us for the R_SVD + Walsh-Hadamard one).
constexpr int kTcMinM = 1;

bool has_perm_scratch(const ActArgs* a) {
  return a->ws != nullptr && a->ws_bytes >= static_cast<size_t>(a->M) * a->K * 2 &&
         (reinterpret_cast<uintptr_t>(a->ws) & 15u) == 0;
}

// bf16 problems with a tensor-core image and block 64 / 128 go to the tensor
// cores (through a permuted copy when the call gave
// scratch for it, else gathering); returns the rest.
cudaError_t launch_tc_subset(std::vector<const ActArgs*>& v, cudaStream_t stream) {
  if (rsvd_path_forced()) return cudaSuccess;
  std::vector<const ActArgs*> rest, perm, g[2][3], t[2][3];
  for (const ActArgs* a : v) {
    if (a->rot_tc == nullptr || (a->block != 64 && a->block != 128) || a->M < kTcMinM) {
      rest.push_back(a);
      continue;
    }
    const int mode = a->xq == nullptr ? kRotateOnly : a->dynamic ? kDynamic : kTable;
    const int bi = a->block == 64 ? 0 : 1;
    if (has_perm_scratch(a)) {
      perm.push_back(a);
      t[bi][mode].push_back(a);
    } else {
      g[bi][mode].push_back(a);
    }
  }
  cudaError_t e = launch_permute(perm, stream);
  if (e == cudaSuccess) e = launch_tc_mode<64, kTable, true>(t[0][kTable], stream);
  if (e == cudaSuccess) e = launch_tc_mode<64, kDynamic, true>(t[0][kDynamic], stream);
  if (e == cudaSuccess) e = launch_tc_mode<64, kRotateOnly, true>(t[0][kRotateOnly], stream);
  if (e == cudaSuccess) e = launch_tc_mode<128, kTable, true>(t[1][kTable], stream);
  if (e == cudaSuccess) e = launch_tc_mode<128, kDynamic, true>(t[1][kDynamic], stream);
  if (e == cudaSuccess) e = launch_tc_mode<128, kRotateOnly, true>(t[1][kRotateOnly], stream);
  if (e == cudaSuccess) e = launch_tc_mode<64, kTable, false>(g[0][kTable], stream);
  if (e == cudaSuccess) e = launch_tc_mode<64, kDynamic, false>(g[0][kDynamic], stream);
  if (e == cudaSuccess) e = launch_tc_mode<64, kRotateOnly, false>(g[0][kRotateOnly], stream);
  if (e == cudaSuccess) e = launch_tc_mode<128, kTable, false>(g[1][kTable], stream);
  if (e == cudaSuccess) e = launch_tc_mode<128, kDynamic, false>(g[1][kDynamic], stream);
  if (e == cudaSuccess) e = launch_tc_mode<128, kRotateOnly, false>(g[1][kRotateOnly], stream);
  v.swap(rest);
  return e;
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
  cudaError_t e = launch_tc_subset(bf, stream);     // leaves the rest in bf
  if (e == cudaSuccess && !bf.empty()) e = launch_dtype<__nv_bfloat16>(bf, stream);
  if (e == cudaSuccess && !f32.empty()) e = launch_dtype<float>(f32, stream);
  // the int8 images the CUDA-core routes did not write
  if (e == cudaSuccess) {
    std::vector<const ActArgs*> rest(bf);
    rest.insert(rest.end(), f32.begin(), f32.end());
    e = launch_expand(rest, stream);
  }
  return e;
}

cudaError_t launch_rotate_quant(const ActArgs& a, cudaStream_t stream) {
  return launch_rotate_quant_batch(&a, 1, stream);
}

cudaError_t launch_quant_rows_batch(const QuantArgs* as, int n, cudaStream_t stream) {
  for (int i0 = 0; i0 < n; i0 += kMaxBatch) {
    const int m = std::min(kMaxBatch, n - i0);
    QuantBatch b;
    std::memset(&b, 0, sizeof(b));
    b.n = m;
    long long rows = 0;
    for (int i = 0; i < m; ++i) {
      const QuantArgs& a = as[i0 + i];
      b.j[i] = QuantJob{a.xr, a.table, a.step_dev, a.q_out, a.s_out, a.K, a.qmin, a.qmax,
                        a.dynamic, a.T, a.Lcount, a.step_host, a.layer, a.bits == 8 ? 8 : 4};
      b.row_start[i] = static_cast<int>(rows);
      rows += std::max(0, a.rows);
    }
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    b.row_start[m] = static_cast<int>(rows);
    if (rows == 0) continue;
    quant_rows_kernel<<<static_cast<unsigned>(rows), kThreads, 0, stream>>>(b, device_error_word());
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_quant_rows(const QuantArgs& a, cudaStream_t stream) {
  return launch_quant_rows_batch(&a, 1, stream);
}

}  // namespace qvla
