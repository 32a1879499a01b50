// C ABI of the rotated W4A4 linear layer: argument validation, status codes,
// the per-device error word, and the offline pack orchestration (zigzag
// permutation and R_SVD eigensolve on the host, everything else on the GPU).
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

#include "qvla_common.cuh"
#include "qvla_internal.h"

// Device error word: kernels OR QVLA_DEVERR_* bits into it.
__device__ unsigned int g_qvla_error_word = 0u;

namespace qvla {

unsigned int* device_error_word() {
  static std::mutex mu;
  static unsigned int* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_qvla_error_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  return addr[dev];
}

namespace {
// One warp: holds tensor memory and an mbarrier that nothing ever arrives on,
// waits on it with the production bounded wait, gives up after limit_ns,
// then frees its tensor memory and returns.  The wait expiring is the
// expected outcome: it must set QVLA_DEVERR_TIMEOUT and nothing else.
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(uint64_t limit_ns,
                                                                   unsigned int* err) {
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  tmem_alloc(&tmem_slot, 32);
  tmem_relinquish();
  tc_fence_before();
  __syncwarp();
  tc_fence_after();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, limit_ns);
  __syncwarp();
  tc_fence_after();
  tmem_dealloc(tmem_slot, 32);
}
}  // namespace

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("QVLA_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_block(int b) { return b == 32 || b == 64 || b == 128 || b == 256; }

qvla_status check_shape(int N, int K, int block) {
  if (N <= 0 || K <= 0 || !valid_block(block)) return QVLA_ERR_SHAPE;
  if (K % block != 0 || K > QVLA_MAX_K) return QVLA_ERR_SHAPE;
  return QVLA_OK;
}

qvla_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QVLA_OK : QVLA_ERR_CUDA; }

qvla_status check_linear(const qvla_packed_linear* L, bool need_weights) {
  if (!L) return QVLA_ERR_ARG;
  qvla_status st = check_shape(L->N, L->K, L->block);
  if (st != QVLA_OK) return st;
  // rot == NULL: Hadamard-only linear (R_SVD = I), which has no tensor-core image
  if (!L->perm) return QVLA_ERR_ARG;
  if (need_weights && (!L->wq || !L->w_scale)) return QVLA_ERR_ARG;
  if (!aligned16(L->perm) || (L->rot && !aligned16(L->rot))) return QVLA_ERR_ALIGN;
  if (L->rot_tc && !aligned16(L->rot_tc)) return QVLA_ERR_ALIGN;
  if (need_weights && (!aligned16(L->wq) || !aligned16(L->w_scale))) return QVLA_ERR_ALIGN;
  if (L->bias && !aligned16(L->bias)) return QVLA_ERR_ALIGN;
  return QVLA_OK;
}

qvla_status check_scale(qvla_scale_mode mode, const float* table, int T, int Lcount,
                        const int32_t* step_dev, int step_host, int layer) {
  if (mode == QVLA_SCALE_DYNAMIC) return QVLA_OK;
  if (mode != QVLA_SCALE_TABLE) return QVLA_ERR_ARG;
  if (!table || T <= 0 || Lcount <= 0) return QVLA_ERR_ARG;
  if (layer < 0 || layer >= Lcount) return QVLA_ERR_STEP_RANGE;
  if (!step_dev && (step_host < 0 || step_host >= T)) return QVLA_ERR_STEP_RANGE;
  return QVLA_OK;
}

// ------------------------------------------------------------ host eigensolve
// Cyclic Jacobi eigen-decomposition of a symmetric n x n matrix (fp64).
// Each rotation in the (p, q) plane zeroes A[p][q]:
//   theta = (A[q][q] - A[p][p]) / (2 A[p][q]),
//   t = sign(theta) / (|theta| + sqrt(theta^2 + 1)),  c = 1/sqrt(1+t^2), s = t c,
//   A[p][p] -= t A[p][q],  A[q][q] += t A[p][q],
//   rows/columns p, q and the accumulated eigenvector columns rotate by (c, s).
// Sweeps stop when the off-diagonal Frobenius norm is below 1e-15 ||A||_F.
void jacobi_eig(std::vector<double>& A, int n, std::vector<double>& V) {
  V.assign(static_cast<size_t>(n) * n, 0.0);
  for (int i = 0; i < n; ++i) V[static_cast<size_t>(i) * n + i] = 1.0;
  double frob = 0.0;
  for (double a : A) frob += a * a;
  frob = std::sqrt(frob);
  if (frob == 0.0) return;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = p + 1; q < n; ++q) off += 2.0 * A[static_cast<size_t>(p) * n + q] * A[static_cast<size_t>(p) * n + q];
    if (std::sqrt(off) <= 1e-15 * frob) break;
    for (int p = 0; p < n - 1; ++p) {
      for (int q = p + 1; q < n; ++q) {
        const double apq = A[static_cast<size_t>(p) * n + q];
        if (apq == 0.0) continue;
        const double app = A[static_cast<size_t>(p) * n + p];
        const double aqq = A[static_cast<size_t>(q) * n + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0);
        const double s = t * c;
        for (int k = 0; k < n; ++k) {
          if (k == p || k == q) continue;
          const double akp = A[static_cast<size_t>(k) * n + p];
          const double akq = A[static_cast<size_t>(k) * n + q];
          const double nkp = c * akp - s * akq;
          const double nkq = s * akp + c * akq;
          A[static_cast<size_t>(k) * n + p] = nkp;
          A[static_cast<size_t>(p) * n + k] = nkp;
          A[static_cast<size_t>(k) * n + q] = nkq;
          A[static_cast<size_t>(q) * n + k] = nkq;
        }
        A[static_cast<size_t>(p) * n + p] = app - t * apq;
        A[static_cast<size_t>(q) * n + q] = aqq + t * apq;
        A[static_cast<size_t>(p) * n + q] = 0.0;
        A[static_cast<size_t>(q) * n + p] = 0.0;
        for (int k = 0; k < n; ++k) {
          const double vkp = V[static_cast<size_t>(k) * n + p];
          const double vkq = V[static_cast<size_t>(k) * n + q];
          V[static_cast<size_t>(k) * n + p] = c * vkp - s * vkq;
          V[static_cast<size_t>(k) * n + q] = s * vkp + c * vkq;
        }
      }
    }
  }
}

// R_SVD of one block from its Gram matrix: eigenvectors by descending
// eigenvalue (ties to the lower index), largest-magnitude entry of each
// column made positive (first index on ties).  out is row-major [i][j].
void rsvd_from_gram(const double* G, int b, double* out) {
  std::vector<double> A(G, G + static_cast<size_t>(b) * b), V;
  jacobi_eig(A, b, V);
  std::vector<int> idx(b);
  for (int i = 0; i < b; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](int x, int y) {
    return A[static_cast<size_t>(x) * b + x] > A[static_cast<size_t>(y) * b + y];
  });
  for (int j = 0; j < b; ++j) {
    const int src = idx[j];
    int imax = 0;
    double vmax = -1.0;
    for (int i = 0; i < b; ++i) {
      const double v = std::fabs(V[static_cast<size_t>(i) * b + src]);
      if (v > vmax) {
        vmax = v;
        imax = i;
      }
    }
    const double sg = V[static_cast<size_t>(imax) * b + src] < 0 ? -1.0 : 1.0;
    for (int i = 0; i < b; ++i) out[static_cast<size_t>(i) * b + j] = sg * V[static_cast<size_t>(i) * b + src];
  }
}

// Zigzag permutation from column norms (see qvla_pack_weights).
void zigzag_from_norms(const std::vector<double>& c, int block, std::vector<int32_t>& perm) {
  const int K = static_cast<int>(c.size());
  const int nb = K / block;
  std::vector<int> order(K);
  for (int k = 0; k < K; ++k) order[k] = k;
  std::sort(order.begin(), order.end(), [&](int a, int b) {
    return c[a] > c[b] || (c[a] == c[b] && a < b);
  });
  perm.assign(K, 0);
  for (int r = 0; r < K; ++r) {
    const int rnd = r / nb, pos = r % nb;
    const int blk = (rnd % 2 == 0) ? pos : nb - 1 - pos;
    perm[static_cast<size_t>(blk) * block + rnd] = order[r];
  }
}

size_t pack_ws_bytes(int N, int K, int block) {
  const size_t nb = K / block;
  size_t b = 0;
  b += static_cast<size_t>(K) * 8;                               // norms
  b += nb * block * block * 8;                                   // Gram
  b += nb * block * block * 8;                                   // R_SVD fp64
  b = (b + 255) & ~static_cast<size_t>(255);
  b += static_cast<size_t>(N) * K * 4;                           // W' fp32
  return b;
}

}  // namespace
}  // namespace qvla

using namespace qvla;

// The rotation of qvla_rotate_act_f32 with an optional permuted-copy scratch.
static qvla_status rotate_act_impl(const void* x, qvla_dtype xdt, int M, int ldx,
                                   const qvla_packed_linear* L, float* xr_out, void* perm_ws,
                                   size_t perm_ws_bytes, cudaStream_t stream);

extern "C" {

const char* qvla_status_str(qvla_status s) {
  switch (s) {
    case QVLA_OK: return "ok";
    case QVLA_ERR_ARG: return "invalid argument (null pointer or enum)";
    case QVLA_ERR_SHAPE: return "unsupported shape";
    case QVLA_ERR_ALIGN: return "pointer or pitch not 16-byte aligned";
    case QVLA_ERR_STEP_RANGE: return "denoising step or layer outside the scale table";
    case QVLA_ERR_UNSUPPORTED: return "unsupported device or feature";
    case QVLA_ERR_CUDA: return "CUDA error";
    case QVLA_ERR_DEVICE_FLAG: return "device error word set";
    case QVLA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int qvla_abi_version(void) { return QVLA_ABI_VERSION; }

#ifndef QVLA_SOURCE_SHA256
#define QVLA_SOURCE_SHA256 "unstamped"
#endif
// The build stamps the hash of its inputs here; the prefix lets a build
// script find it in the file without loading the library.
__attribute__((used)) static const char kSourceStamp[] = "QVLA_SOURCE_SHA256=" QVLA_SOURCE_SHA256;

const char* qvla_source_hash(void) { return kSourceStamp + sizeof("QVLA_SOURCE_SHA256=") - 1; }

qvla_status qvla_read_error_word(uint32_t* out, int clear) {
  if (!out) return QVLA_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return QVLA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_qvla_error_word, sizeof(v)) != cudaSuccess) return QVLA_ERR_CUDA;
  *out = v;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_qvla_error_word, &z, sizeof(z)) != cudaSuccess) return QVLA_ERR_CUDA;
  }
  return QVLA_OK;
}

qvla_status qvla_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
  if (limit_ns < 1000ull || limit_ns > 10000000ull) return QVLA_ERR_ARG;
  unsigned int* err = device_error_word();
  if (!err) return QVLA_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
  return cuda_status(cudaGetLastError());
}

qvla_status qvla_packed_sizes(int N, int K, int block, size_t* wq_bytes, size_t* rot_bytes,
                              size_t* rot_tc_bytes, size_t* ws_bytes) {
  qvla_status st = check_shape(N, K, block);
  if (st != QVLA_OK) return st;
  if (K % 32) return QVLA_ERR_SHAPE;
  if (wq_bytes) *wq_bytes = static_cast<size_t>(N) * K / 2;
  if (rot_bytes) *rot_bytes = static_cast<size_t>(K) * block * 4;
  if (rot_tc_bytes)
    *rot_tc_bytes = (block == 64 || block == 128) ? static_cast<size_t>(K) * block * 6 : 0;
  if (ws_bytes) *ws_bytes = pack_ws_bytes(N, K, block);
  return QVLA_OK;
}

qvla_status qvla_rotate_weights_f32(const float* W, int N, int K, int block, const int32_t* perm,
                                    const double* rsvd64, float* Wr_out, cudaStream_t stream) {
  qvla_status st = check_shape(N, K, block);
  if (st != QVLA_OK) return st;
  if (!W || !perm || !rsvd64 || !Wr_out) return QVLA_ERR_ARG;
  if (!aligned16(W) || !aligned16(Wr_out) || !aligned16(perm) || !aligned16(rsvd64))
    return QVLA_ERR_ALIGN;
  return cuda_status(launch_rotate_weights(W, N, K, block, perm, rsvd64, Wr_out, stream));
}

qvla_status qvla_quant_pack_weights_f32(const float* Wr, int N, int K, uint8_t* wq_out,
                                        float* w_scale_out, cudaStream_t stream) {
  if (N <= 0 || K <= 0 || K % 32 || K > QVLA_MAX_K) return QVLA_ERR_SHAPE;
  if (!Wr || !wq_out || !w_scale_out) return QVLA_ERR_ARG;
  if (!aligned16(Wr) || !aligned16(wq_out) || !aligned16(w_scale_out)) return QVLA_ERR_ALIGN;
  QuantArgs a = {};
  a.xr = Wr;
  a.rows = N;
  a.K = K;
  a.qmin = -7;
  a.qmax = 7;
  a.dynamic = 1;
  a.q_out = wq_out;
  a.s_out = w_scale_out;
  return cuda_status(launch_quant_rows(a, stream));
}

// The pack.  hadamard_only: R_SVD = I for every block (no Gram matrices, no
// eigensolve; rot_out and rot_tc_out are not written).
static qvla_status pack_impl(const float* W, int N, int K, int block, const int32_t* perm_in,
                             const double* rsvd_in, bool hadamard_only, int bits, int32_t* perm_out,
                             float* rot_out, uint16_t* rot_tc_out, uint8_t* wq_out,
                             float* w_scale_out, void* workspace, size_t ws_bytes,
                             cudaStream_t stream) {
  qvla_status st = check_shape(N, K, block);
  if (st != QVLA_OK) return st;
  if (K % 32) return QVLA_ERR_SHAPE;
  if (!W || !perm_out || (!rot_out && !hadamard_only) || !wq_out || !w_scale_out)
    return QVLA_ERR_ARG;
  if (!workspace || ws_bytes < pack_ws_bytes(N, K, block)) return QVLA_ERR_WORKSPACE;
  if (!aligned16(W) || !aligned16(perm_out) || (rot_out && !aligned16(rot_out)) ||
      !aligned16(wq_out) || !aligned16(w_scale_out) || !aligned16(workspace))
    return QVLA_ERR_ALIGN;
  const int nb = K / block;
  const size_t bb = static_cast<size_t>(block) * block;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* norms = reinterpret_cast<double*>(ws);
  double* gram = norms + K;
  double* rsvd_dev = gram + nb * bb;
  size_t off = (static_cast<size_t>(K) * 8 + 2 * nb * bb * 8 + 255) & ~static_cast<size_t>(255);
  float* Wr = reinterpret_cast<float*>(ws + off);

  // 1. zigzag permutation
  std::vector<int32_t> perm(K);
  if (perm_in) {
    std::vector<char> seen(K, 0);
    for (int k = 0; k < K; ++k) {
      const int p = perm_in[k];
      if (p < 0 || p >= K || seen[p]) return QVLA_ERR_ARG;
      seen[p] = 1;
      perm[k] = p;
    }
  } else {
    if (launch_column_norms(W, N, K, norms, stream) != cudaSuccess) return QVLA_ERR_CUDA;
    std::vector<double> c(K);
    if (cudaMemcpyAsync(c.data(), norms, K * sizeof(double), cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return QVLA_ERR_CUDA;
    zigzag_from_norms(c, block, perm);
  }
  if (cudaMemcpyAsync(perm_out, perm.data(), K * sizeof(int32_t), cudaMemcpyHostToDevice,
                      stream) != cudaSuccess)
    return QVLA_ERR_CUDA;

  // 2. R_SVD per block
  std::vector<double> rs(nb * bb, 0.0);
  if (hadamard_only) {
    for (int B = 0; B < nb; ++B)
      for (int i = 0; i < block; ++i) rs[B * bb + static_cast<size_t>(i) * block + i] = 1.0;
  } else if (rsvd_in) {
    std::memcpy(rs.data(), rsvd_in, rs.size() * sizeof(double));
  } else {
    if (launch_block_gram(W, N, K, block, perm_out, gram, stream) != cudaSuccess)
      return QVLA_ERR_CUDA;
    std::vector<double> G(nb * bb);
    if (cudaMemcpyAsync(G.data(), gram, G.size() * sizeof(double), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return QVLA_ERR_CUDA;
    unsigned nthreads = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
    nthreads = std::min<unsigned>(nthreads, static_cast<unsigned>(nb));
    std::vector<std::thread> pool;
    for (unsigned t = 0; t < nthreads; ++t)
      pool.emplace_back([&, t]() {
        for (int B = static_cast<int>(t); B < nb; B += static_cast<int>(nthreads))
          rsvd_from_gram(G.data() + B * bb, block, rs.data() + B * bb);
      });
    for (auto& th : pool) th.join();
  }
  std::vector<float> rs32(rs.size());
  for (size_t i = 0; i < rs.size(); ++i) rs32[i] = static_cast<float>(rs[i]);
  if (cudaMemcpyAsync(rsvd_dev, rs.data(), rs.size() * sizeof(double), cudaMemcpyHostToDevice,
                      stream) != cudaSuccess ||
      (!hadamard_only && cudaMemcpyAsync(rot_out, rs32.data(), rs32.size() * sizeof(float),
                                         cudaMemcpyHostToDevice, stream) != cudaSuccess))
    return QVLA_ERR_CUDA;

  if (rot_tc_out && (block == 64 || block == 128)) {
    if (!aligned16(rot_tc_out)) return QVLA_ERR_ALIGN;
    if (launch_rot_tc_image(rsvd_dev, K, block, rot_tc_out, stream) != cudaSuccess)
      return QVLA_ERR_CUDA;
  }

  // 3. W' = fp32(W P R) in fp64, then RTN + packing
  if (launch_rotate_weights(W, N, K, block, perm_out, rsvd_dev, Wr, stream) != cudaSuccess)
    return QVLA_ERR_CUDA;
  QuantArgs q = {};
  q.xr = Wr;
  q.rows = N;
  q.K = K;
  q.qmin = bits == 8 ? -127 : -7;
  q.qmax = bits == 8 ? 127 : 7;
  q.dynamic = 1;
  q.bits = bits;
  q.q_out = wq_out;
  q.s_out = w_scale_out;
  if (launch_quant_rows(q, stream) != cudaSuccess) return QVLA_ERR_CUDA;
  // host staging vectors must outlive the copies
  if (cudaStreamSynchronize(stream) != cudaSuccess) return QVLA_ERR_CUDA;
  return QVLA_OK;
}

qvla_status qvla_pack_weights(const float* W, int N, int K, int block, const int32_t* perm_in,
                              const double* rsvd_in, int32_t* perm_out, float* rot_out,
                              uint16_t* rot_tc_out, uint8_t* wq_out, float* w_scale_out,
                              void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return pack_impl(W, N, K, block, perm_in, rsvd_in, false, 4, perm_out, rot_out, rot_tc_out,
                   wq_out, w_scale_out, workspace, ws_bytes, stream);
}

qvla_status qvla_gptq_hessian_host(const float* xr, int T, int K, double* H_out) {
  if (T <= 0 || K <= 0 || K > 4096) return QVLA_ERR_SHAPE;
  if (!xr || !H_out) return QVLA_ERR_ARG;
  std::vector<double> H;
  gptq_hessian(xr, T, K, H);
  std::memcpy(H_out, H.data(), H.size() * sizeof(double));
  return QVLA_OK;
}

qvla_status qvla_gptq_quantize_host(const float* Wr, int N, int K, const double* H, double damp,
                                    const double* u_in, int8_t* q_out, float* s_out) {
  if (N <= 0 || K <= 0 || K > 4096) return QVLA_ERR_SHAPE;
  if (!Wr || !q_out || !s_out || (!H && !u_in) || !(damp >= 0.0)) return QVLA_ERR_ARG;
  std::vector<double> U;
  std::vector<char> dead;
  const double* u = u_in;
  if (!u) {
    if (!gptq_inverse_factor(H, K, damp, U, dead)) return QVLA_ERR_ARG;
    u = U.data();
  }
  gptq_quantize_rows(Wr, N, K, u, dead.empty() ? nullptr : dead.data(), 7, q_out, s_out);
  return QVLA_OK;
}

qvla_status qvla_pack_weights_gptq(const float* W, int N, int K, int block, const void* x_cal,
                                   qvla_dtype xdt, int T, double damp, const int32_t* perm_in,
                                   const double* rsvd_in, const double* u_in, int32_t* perm_out,
                                   float* rot_out, uint16_t* rot_tc_out, uint8_t* wq_out,
                                   float* w_scale_out, void* workspace, size_t ws_bytes,
                                   void* cal_workspace, size_t cal_ws_bytes,
                                   cudaStream_t stream) {
  if (K > 4096) return QVLA_ERR_SHAPE;                 // fp64 K x K work on the host
  if (!u_in) {
    if (!x_cal || T <= 0 || (xdt != QVLA_DTYPE_F32 && xdt != QVLA_DTYPE_BF16))
      return QVLA_ERR_ARG;
    if (!cal_workspace || cal_ws_bytes < static_cast<size_t>(T) * K * 4) return QVLA_ERR_WORKSPACE;
  }
  // 1. permutation, R_SVD, rotated weights (and RTN codes, replaced below)
  qvla_status st = pack_impl(W, N, K, block, perm_in, rsvd_in, false, 4, perm_out, rot_out,
                             rot_tc_out, wq_out, w_scale_out, workspace, ws_bytes, stream);
  if (st != QVLA_OK) return st;
  const int nb = K / block;
  const size_t bb = static_cast<size_t>(block) * block;
  const size_t off = (static_cast<size_t>(K) * 8 + 2 * nb * bb * 8 + 255) & ~static_cast<size_t>(255);
  std::vector<float> Wr(static_cast<size_t>(N) * K);
  if (cudaStreamSynchronize(stream) != cudaSuccess ||
      cudaMemcpy(Wr.data(), static_cast<uint8_t*>(workspace) + off, Wr.size() * 4,
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return QVLA_ERR_CUDA;
  // 2. the inverse factor of the damped Hessian of the rotated calibration rows
  std::vector<double> U;
  std::vector<char> dead;
  const double* u = u_in;
  if (!u) {
    qvla_packed_linear Lc = {N, K, block, perm_out, rot_out, nullptr, wq_out, w_scale_out, nullptr};
    float* xr_dev = static_cast<float*>(cal_workspace);
    if ((st = qvla_rotate_act_f32(x_cal, xdt, T, K, &Lc, xr_dev, stream)) != QVLA_OK) return st;
    std::vector<float> xr(static_cast<size_t>(T) * K);
    if (cudaStreamSynchronize(stream) != cudaSuccess ||
        cudaMemcpy(xr.data(), xr_dev, xr.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return QVLA_ERR_CUDA;
    std::vector<double> H;
    gptq_hessian(xr.data(), T, K, H);
    if (!gptq_inverse_factor(H.data(), K, damp, U, dead)) return QVLA_ERR_ARG;
    u = U.data();
  }
  // 3. GPTQ codes, packed two per byte
  std::vector<int8_t> q(static_cast<size_t>(N) * K);
  std::vector<float> s(N);
  gptq_quantize_rows(Wr.data(), N, K, u, dead.empty() ? nullptr : dead.data(), 7, q.data(),
                     s.data());
  std::vector<uint8_t> packed(static_cast<size_t>(N) * K / 2);
  for (size_t i = 0; i < packed.size(); ++i)
    packed[i] = static_cast<uint8_t>((q[2 * i] & 15) | ((q[2 * i + 1] & 15) << 4));
  if (cudaMemcpyAsync(wq_out, packed.data(), packed.size(), cudaMemcpyHostToDevice, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(w_scale_out, s.data(), s.size() * 4, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return QVLA_ERR_CUDA;
  return QVLA_OK;
}

qvla_status qvla_pack_weights_w8(const float* W, int N, int K, int block, const int32_t* perm_in,
                                 const double* rsvd_in, int32_t* perm_out, float* rot_out,
                                 uint16_t* rot_tc_out, uint8_t* wq_out, float* w_scale_out,
                                 void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return pack_impl(W, N, K, block, perm_in, rsvd_in, false, 8, perm_out, rot_out, rot_tc_out,
                   wq_out, w_scale_out, workspace, ws_bytes, stream);
}

qvla_status qvla_pack_weights_hadamard(const float* W, int N, int K, int block,
                                       const int32_t* perm_in, int32_t* perm_out,
                                       uint16_t* rot_tc_out, uint8_t* wq_out,
                                       float* w_scale_out, void* workspace, size_t ws_bytes,
                                       cudaStream_t stream) {
  return pack_impl(W, N, K, block, perm_in, nullptr, true, 4, perm_out, nullptr, rot_tc_out,
                   wq_out, w_scale_out, workspace, ws_bytes, stream);
}

// Validates one rotate-quantise call and fills its launch arguments.
static qvla_status prepare_act(const void* x, qvla_dtype xdt, int M, int ldx,
                               const qvla_packed_linear* L, qvla_scale_mode mode,
                               const float* table, int T, int Lcount, const int32_t* step_dev,
                               int step_host, int layer, uint8_t* xq, float* s_x,
                               ActArgs* out) {
  qvla_status st = check_linear(L, false);
  if (st != QVLA_OK) return st;
  if (M < 0) return QVLA_ERR_SHAPE;
  if (xdt != QVLA_DTYPE_F32 && xdt != QVLA_DTYPE_BF16) return QVLA_ERR_ARG;
  if ((st = check_scale(mode, table, T, Lcount, step_dev, step_host, layer)) != QVLA_OK) return st;
  *out = ActArgs{};
  out->M = M;
  if (M == 0) return QVLA_OK;
  if (!x || !xq || !s_x) return QVLA_ERR_ARG;
  if (ldx < L->K) return QVLA_ERR_SHAPE;
  const size_t esz = xdt == QVLA_DTYPE_F32 ? 4 : 2;
  if (!aligned16(x) || (ldx * esz) % 16 || !aligned16(xq) || !aligned16(s_x)) return QVLA_ERR_ALIGN;
  ActArgs& a = *out;
  a.x = x;
  a.xdt = xdt;
  a.M = M;
  a.ldx = ldx;
  a.K = L->K;
  a.block = L->block;
  a.perm = L->perm;
  a.rot = L->rot;
  a.rot_tc = (L->rot_tc && (L->block == 64 || L->block == 128)) ? L->rot_tc : nullptr;
  a.dynamic = mode == QVLA_SCALE_DYNAMIC;
  a.table = table;
  a.T = T;
  a.Lcount = Lcount;
  a.step_dev = step_dev;
  a.step_host = step_host;
  a.layer = layer;
  a.xq = xq;
  a.s_x = s_x;
  return QVLA_OK;
}

qvla_status qvla_rotate_quant_act(const void* x, qvla_dtype xdt, int M, int ldx,
                                  const qvla_packed_linear* L, qvla_scale_mode mode,
                                  const float* table, int T, int Lcount, const int32_t* step_dev,
                                  int step_host, int layer, uint8_t* xq, float* s_x,
                                  void* workspace, size_t ws_bytes, cudaStream_t stream) {
  ActArgs a;
  qvla_status st = prepare_act(x, xdt, M, ldx, L, mode, table, T, Lcount, step_dev, step_host,
                               layer, xq, s_x, &a);
  if (st != QVLA_OK || M == 0) return st;
  a.ws = workspace;
  a.ws_bytes = ws_bytes;
  return cuda_status(launch_rotate_quant(a, stream));
}

qvla_status qvla_rotate_quant_workspace_bytes(int M, int K, int block, qvla_dtype xdt,
                                              size_t* bytes) {
  if (!bytes) return QVLA_ERR_ARG;
  if (M < 0 || K <= 0 || K > QVLA_MAX_K || !valid_block(block) || K % block) return QVLA_ERR_SHAPE;
  const bool tc = xdt == QVLA_DTYPE_BF16 && (block == 64 || block == 128) && M > 0;
  // the permuted copy of x, then (DYNAMIC) the row maxima of up to K / block
  // CTAs per token
  *bytes = tc ? static_cast<size_t>(M) * K * 2 + static_cast<size_t>(M) * (K / block) * 4 : 0;
  return QVLA_OK;
}

}  // extern "C"

// Scratch of qvla_rotate_quant_act_noalloc, for callers that cannot allocate
// device memory while they run: a fixed array in the library's module, one per
// device that loads it, held until the process exits.  Host code must not pass
// the symbol itself to a kernel (in host code it is only a stand-in for the
// device array); the entry point looks up its device address per device.
static __device__ __align__(256) unsigned char g_qvla_noalloc_scratch[QVLA_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array for the current device, looked up once
// per device with that device current.
qvla_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QVLA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_qvla_noalloc_scratch) != cudaSuccess || p == nullptr)
      return QVLA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return QVLA_OK;
}

}  // namespace

extern "C" {

qvla_status qvla_rotate_quant_act_noalloc(const void* x, qvla_dtype xdt, int M, int ldx,
                                          const qvla_packed_linear* L, qvla_scale_mode mode,
                                          const float* table, int T, int Lcount,
                                          const int32_t* step_dev, int step_host, int layer,
                                          uint8_t* xq, float* s_x, cudaStream_t stream) {
  ActArgs a;
  qvla_status st = prepare_act(x, xdt, M, ldx, L, mode, table, T, Lcount, step_dev, step_host,
                               layer, xq, s_x, &a);
  if (st != QVLA_OK || M == 0) return st;
  size_t need = 0;
  if ((st = qvla_rotate_quant_workspace_bytes(M, L->K, L->block, xdt, &need)) != QVLA_OK)
    return st;
  // the permuted copy must fit; the row maxima of the two-launch DYNAMIC
  // route are used only if they fit as well (the route checks the size)
  if (need > 0 && static_cast<size_t>(M) * L->K * 2 > QVLA_NOALLOC_SCRATCH_BYTES)
    return QVLA_ERR_WORKSPACE;
  if (need > 0) {
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != QVLA_OK) return st;
    a.ws = scratch;
    a.ws_bytes = QVLA_NOALLOC_SCRATCH_BYTES;
  }
  return cuda_status(launch_rotate_quant(a, stream));
}

qvla_status qvla_rotate_quant_act_batched(const qvla_linear_problem* probs, int n,
                                          cudaStream_t stream) {
  if (n < 0 || (n > 0 && !probs)) return QVLA_ERR_ARG;
  std::vector<ActArgs> v(n);
  for (int i = 0; i < n; ++i) {
    const qvla_linear_problem& p = probs[i];
    qvla_status st = prepare_act(p.x, static_cast<qvla_dtype>(p.xdt), p.M, p.ldx, p.L,
                                 static_cast<qvla_scale_mode>(p.mode), p.table, p.T, p.Lcount,
                                 p.step_dev, p.step_host, p.layer, p.xq, p.s_x, &v[i]);
    if (st != QVLA_OK) return st;
    v[i].ws = p.workspace;
    v[i].ws_bytes = p.ws_bytes;
    if (p.M > 0 && p.xq8 && !aligned16(p.xq8)) return QVLA_ERR_ALIGN;
    v[i].xq8 = p.M > 0 ? p.xq8 : nullptr;
  }
  // the problems run concurrently: their scratch ranges must be disjoint
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(v[i].ws), b0 = reinterpret_cast<uintptr_t>(v[j].ws);
      if (!a0 || !b0) continue;
      if (a0 < b0 + v[j].ws_bytes && b0 < a0 + v[i].ws_bytes) return QVLA_ERR_ARG;
    }
  return cuda_status(launch_rotate_quant_batch(v.data(), n, stream));
}

qvla_status qvla_rotate_quant_a8_workspace_bytes(int M, int K, size_t* bytes) {
  if (!bytes) return QVLA_ERR_ARG;
  if (M < 0 || K <= 0 || K > QVLA_MAX_K) return QVLA_ERR_SHAPE;
  *bytes = static_cast<size_t>(M) * K * 6;
  return QVLA_OK;
}

qvla_status qvla_rotate_quant_act_a8(const void* x, qvla_dtype xdt, int M, int ldx,
                                     const qvla_packed_linear* L, int8_t* xq8, float* s_x,
                                     void* workspace, size_t ws_bytes, cudaStream_t stream) {
  qvla_status st = check_linear(L, false);
  if (st != QVLA_OK) return st;
  if (M < 0) return QVLA_ERR_SHAPE;
  if (M == 0) return QVLA_OK;
  if (!xq8 || !s_x) return QVLA_ERR_ARG;
  if (!aligned16(xq8) || !aligned16(s_x)) return QVLA_ERR_ALIGN;
  const size_t xr_bytes = static_cast<size_t>(M) * L->K * 4;
  if (!workspace || ws_bytes < xr_bytes) return QVLA_ERR_WORKSPACE;
  float* xr = static_cast<float*>(workspace);
  // 1. the rotation (fp32 x' into the workspace; the permuted copy of x that
  // the tensor-core route reads goes after it when the workspace has room)
  const size_t perm_bytes = static_cast<size_t>(M) * L->K * 2;
  void* perm_ws = ws_bytes >= xr_bytes + perm_bytes ? static_cast<uint8_t*>(workspace) + xr_bytes : nullptr;
  if ((st = rotate_act_impl(x, xdt, M, ldx, L, xr, perm_ws, perm_ws ? perm_bytes : 0, stream)) !=
      QVLA_OK)
    return st;
  // 2. per-token dynamic 8-bit RTN
  QuantArgs q = {};
  q.xr = xr;
  q.rows = M;
  q.K = L->K;
  q.qmin = -128;
  q.qmax = 127;
  q.dynamic = 1;
  q.bits = 8;
  q.q_out = reinterpret_cast<uint8_t*>(xq8);
  q.s_out = s_x;
  return cuda_status(launch_quant_rows(q, stream));
}

qvla_status qvla_rotate_quant_act_a8_batched(const qvla_linear_problem* probs, int n,
                                             cudaStream_t stream) {
  if (n < 0 || (n > 0 && !probs)) return QVLA_ERR_ARG;
  std::vector<ActArgs> acts;
  std::vector<QuantArgs> quants;
  std::vector<std::pair<uintptr_t, size_t>> ranges;
  for (int i = 0; i < n; ++i) {
    const qvla_linear_problem& p = probs[i];
    qvla_status st = check_linear(p.L, false);
    if (st != QVLA_OK) return st;
    if (p.M < 0) return QVLA_ERR_SHAPE;
    if (p.xdt != QVLA_DTYPE_F32 && p.xdt != QVLA_DTYPE_BF16) return QVLA_ERR_ARG;
    if (p.M == 0) continue;
    const int K = p.L->K;
    if (!p.x || !p.xq8 || !p.s_x) return QVLA_ERR_ARG;
    if (p.ldx < K) return QVLA_ERR_SHAPE;
    const size_t esz = p.xdt == QVLA_DTYPE_F32 ? 4 : 2;
    if (!aligned16(p.x) || (p.ldx * esz) % 16 || !aligned16(p.xq8) || !aligned16(p.s_x) ||
        !aligned16(p.workspace))
      return QVLA_ERR_ALIGN;
    const size_t xr_bytes = static_cast<size_t>(p.M) * K * 4, perm_bytes = static_cast<size_t>(p.M) * K * 2;
    if (!p.workspace || p.ws_bytes < xr_bytes) return QVLA_ERR_WORKSPACE;
    ranges.push_back({reinterpret_cast<uintptr_t>(p.workspace), p.ws_bytes});
    // the rotation into the workspace (fp32 rows; the permuted copy of x
    // after them when there is room), then the 8-bit quantisation of the rows
    ActArgs a = {};
    a.x = p.x;
    a.xdt = static_cast<qvla_dtype>(p.xdt);
    a.M = p.M;
    a.ldx = p.ldx;
    a.K = K;
    a.block = p.L->block;
    a.perm = p.L->perm;
    a.rot = p.L->rot;
    a.rot_tc = (p.L->rot_tc && (p.L->block == 64 || p.L->block == 128)) ? p.L->rot_tc : nullptr;
    a.dynamic = 1;
    a.xr_out = static_cast<float*>(p.workspace);
    if (p.ws_bytes >= xr_bytes + perm_bytes) {
      a.ws = static_cast<uint8_t*>(p.workspace) + xr_bytes;
      a.ws_bytes = perm_bytes;
    }
    acts.push_back(a);
    QuantArgs q = {};
    q.xr = a.xr_out;
    q.rows = p.M;
    q.K = K;
    q.qmin = -128;
    q.qmax = 127;
    q.dynamic = 1;
    q.bits = 8;
    q.q_out = reinterpret_cast<uint8_t*>(p.xq8);
    q.s_out = p.s_x;
    quants.push_back(q);
  }
  // the problems run concurrently: their workspaces must be disjoint
  for (size_t i = 0; i < ranges.size(); ++i)
    for (size_t j = i + 1; j < ranges.size(); ++j)
      if (ranges[i].first < ranges[j].first + ranges[j].second &&
          ranges[j].first < ranges[i].first + ranges[i].second)
        return QVLA_ERR_ARG;
  if (acts.empty()) return QVLA_OK;
  cudaError_t e = launch_rotate_quant_batch(acts.data(), static_cast<int>(acts.size()), stream);
  if (e == cudaSuccess) e = launch_quant_rows_batch(quants.data(), static_cast<int>(quants.size()), stream);
  return cuda_status(e);
}

qvla_status qvla_rotate_act_f32(const void* x, qvla_dtype xdt, int M, int ldx,
                                const qvla_packed_linear* L, float* xr_out, cudaStream_t stream) {
  return rotate_act_impl(x, xdt, M, ldx, L, xr_out, nullptr, 0, stream);
}

}  // extern "C"

// The rotation alone; perm_ws (or NULL) holds the permuted copy of x that the
// tensor-core route reads through TMA.
static qvla_status rotate_act_impl(const void* x, qvla_dtype xdt, int M, int ldx,
                                   const qvla_packed_linear* L, float* xr_out, void* perm_ws,
                                   size_t perm_ws_bytes, cudaStream_t stream) {
  qvla_status st = check_linear(L, false);
  if (st != QVLA_OK) return st;
  if (M < 0) return QVLA_ERR_SHAPE;
  if (xdt != QVLA_DTYPE_F32 && xdt != QVLA_DTYPE_BF16) return QVLA_ERR_ARG;
  if (M == 0) return QVLA_OK;
  if (!x || !xr_out) return QVLA_ERR_ARG;
  if (ldx < L->K) return QVLA_ERR_SHAPE;
  const size_t esz = xdt == QVLA_DTYPE_F32 ? 4 : 2;
  if (!aligned16(x) || (ldx * esz) % 16 || !aligned16(xr_out)) return QVLA_ERR_ALIGN;
  ActArgs a = {};
  a.x = x;
  a.xdt = xdt;
  a.M = M;
  a.ldx = ldx;
  a.K = L->K;
  a.block = L->block;
  a.perm = L->perm;
  a.rot = L->rot;
  a.rot_tc = (L->rot_tc && (L->block == 64 || L->block == 128)) ? L->rot_tc : nullptr;
  a.dynamic = 1;
  a.xr_out = xr_out;
  a.ws = perm_ws;
  a.ws_bytes = perm_ws_bytes;
  return cuda_status(launch_rotate_quant(a, stream));
}

extern "C" {

qvla_status qvla_quant_act_f32(const float* xr, int M, int K, qvla_scale_mode mode,
                               const float* table, int T, int Lcount, const int32_t* step_dev,
                               int step_host, int layer, uint8_t* xq, float* s_x,
                               cudaStream_t stream) {
  if (M < 0 || K <= 0 || K % 32 || K > QVLA_MAX_K) return QVLA_ERR_SHAPE;
  qvla_status st = check_scale(mode, table, T, Lcount, step_dev, step_host, layer);
  if (st != QVLA_OK) return st;
  if (M == 0) return QVLA_OK;
  if (!xr || !xq || !s_x) return QVLA_ERR_ARG;
  if (!aligned16(xr) || !aligned16(xq) || !aligned16(s_x)) return QVLA_ERR_ALIGN;
  QuantArgs a = {};
  a.xr = xr;
  a.rows = M;
  a.K = K;
  a.qmin = -8;
  a.qmax = 7;
  a.dynamic = mode == QVLA_SCALE_DYNAMIC;
  a.table = table;
  a.T = T;
  a.Lcount = Lcount;
  a.step_dev = step_dev;
  a.step_host = step_host;
  a.layer = layer;
  a.q_out = xq;
  a.s_out = s_x;
  return cuda_status(launch_quant_rows(a, stream));
}

// Validates one GEMM call and fills its launch arguments.
static qvla_status prepare_gemm(const uint8_t* xq, const float* s_x, int M,
                                const qvla_packed_linear* L, void* y, int ldy, int32_t* acc,
                                int split_k, GemmArgs* out) {
  qvla_status st = check_linear(L, true);
  if (st != QVLA_OK) return st;
  if (M < 0) return QVLA_ERR_SHAPE;
  if (L->K % 32) return QVLA_ERR_SHAPE;
  *out = GemmArgs{};
  out->M = M;
  if (M == 0) return QVLA_OK;
  if (!xq) return QVLA_ERR_ARG;
  if (!aligned16(xq)) return QVLA_ERR_ALIGN;
  if (y) {
    if (!s_x) return QVLA_ERR_ARG;
    if (ldy < L->N) return QVLA_ERR_SHAPE;
    if (!aligned16(s_x) || !aligned16(y) || (static_cast<size_t>(ldy) * 2) % 16)
      return QVLA_ERR_ALIGN;
  } else {
    if (!acc) return QVLA_ERR_ARG;
    if (!aligned16(acc)) return QVLA_ERR_ALIGN;
  }
  const int nkt = (L->K + 255) / 256;
  if (split_k != 0 && split_k != 1 && split_k != 2 && split_k != 4 && split_k != 8 &&
      split_k != 16)
    return QVLA_ERR_ARG;
  if (split_k > nkt) return QVLA_ERR_SHAPE;
  GemmArgs& g = *out;
  g.xq = xq;
  g.s_x = s_x;
  g.N = L->N;
  g.K = L->K;
  g.wq = L->wq;
  g.w_scale = L->w_scale;
  g.bias = L->bias;
  g.y = y;
  g.ldy = ldy;
  g.acc = acc;
  g.split_k = split_k;
  return QVLA_OK;
}

static qvla_status check_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return QVLA_ERR_CUDA;
  return major == 10 ? QVLA_OK : QVLA_ERR_UNSUPPORTED;
}

static qvla_status gemm_common(const uint8_t* xq, const float* s_x, int M,
                               const qvla_packed_linear* L, void* y, int ldy, int32_t* acc,
                               int split_k, cudaStream_t stream) {
  GemmArgs g;
  qvla_status st = prepare_gemm(xq, s_x, M, L, y, ldy, acc, split_k, &g);
  if (st != QVLA_OK || M == 0) return st;
  if ((st = check_sm100()) != QVLA_OK) return st;
  return cuda_status(launch_w4a4_gemm(g, stream));
}

qvla_status qvla_w4a4_gemm_batched(const qvla_linear_problem* probs, int n, int split_k,
                                   cudaStream_t stream) {
  if (n < 0 || (n > 0 && !probs)) return QVLA_ERR_ARG;
  std::vector<GemmArgs> v(n);
  for (int i = 0; i < n; ++i) {
    const qvla_linear_problem& p = probs[i];
    if (p.M > 0 && !p.y) return QVLA_ERR_ARG;
    qvla_status st = prepare_gemm(p.xq, p.s_x, p.M, p.L, p.y, p.ldy, nullptr, split_k, &v[i]);
    if (st != QVLA_OK) return st;
    if (p.M > 0 && p.xq8 && !aligned16(p.xq8)) return QVLA_ERR_ALIGN;
    v[i].xq8 = p.M > 0 ? p.xq8 : nullptr;
  }
  if (n == 0) return QVLA_OK;
  qvla_status st = check_sm100();
  if (st != QVLA_OK) return st;
  return cuda_status(launch_w4a4_gemm_batch(v.data(), n, split_k, stream));
}

static qvla_status w8a8_common(const int8_t* xq8, const float* s_x, int M,
                               const qvla_packed_linear* L, void* y, int ldy, int32_t* acc,
                               cudaStream_t stream) {
  GemmArgs g;
  qvla_status st = prepare_gemm(reinterpret_cast<const uint8_t*>(xq8), s_x, M, L, y, ldy, acc, 0,
                                &g);
  if (st != QVLA_OK || M == 0) return st;
  if ((st = check_sm100()) != QVLA_OK) return st;
  return cuda_status(launch_w8a8_gemm(g, stream));
}

qvla_status qvla_w8a8_gemm(const int8_t* xq8, const float* s_x, int M,
                           const qvla_packed_linear* L, void* y, int ldy, cudaStream_t stream) {
  if (M > 0 && !y) return QVLA_ERR_ARG;
  return w8a8_common(xq8, s_x, M, L, y, ldy, nullptr, stream);
}

qvla_status qvla_w8a8_gemm_s32(const int8_t* xq8, int M, const qvla_packed_linear* L,
                               int32_t* acc, cudaStream_t stream) {
  return w8a8_common(xq8, nullptr, M, L, nullptr, 0, acc, stream);
}

qvla_status qvla_w8a8_gemm_batched(const qvla_linear_problem* probs, int n, cudaStream_t stream) {
  if (n < 0 || (n > 0 && !probs)) return QVLA_ERR_ARG;
  std::vector<GemmArgs> v(n);
  for (int i = 0; i < n; ++i) {
    const qvla_linear_problem& p = probs[i];
    if (p.M > 0 && !p.y) return QVLA_ERR_ARG;
    qvla_status st = prepare_gemm(reinterpret_cast<const uint8_t*>(p.xq8), p.s_x, p.M, p.L, p.y,
                                  p.ldy, nullptr, 0, &v[i]);
    if (st != QVLA_OK) return st;
  }
  if (n == 0) return QVLA_OK;
  qvla_status st = check_sm100();
  if (st != QVLA_OK) return st;
  return cuda_status(launch_w8a8_gemm_batch(v.data(), n, stream));
}

qvla_status qvla_w4a4_gemm(const uint8_t* xq, const float* s_x, int M,
                           const qvla_packed_linear* L, void* y, int ldy, int split_k,
                           cudaStream_t stream) {
  if (M > 0 && !y) return QVLA_ERR_ARG;
  return gemm_common(xq, s_x, M, L, y, ldy, nullptr, split_k, stream);
}

qvla_status qvla_w4a4_gemm_s32(const uint8_t* xq, int M, const qvla_packed_linear* L,
                               int32_t* acc, int split_k, cudaStream_t stream) {
  return gemm_common(xq, nullptr, M, L, nullptr, 0, acc, split_k, stream);
}

}  // extern "C"
