// Internal (C++) launch interfaces shared by the C-ABI layer and the kernels'
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <vector>
#include <stdint.h>

#include "../../include/qvla.h"

namespace qvla {

// Device error word of the current device (lazily resolved symbol address).
unsigned int* device_error_word();

// Programmatic dependent launch on/off (environment QVLA_PDL=0 turns it off).
bool pdl_enabled();

// Runs `set` (kernel attribute calls, which bind to the current device only)
// once per device: bit d of `done` records device d.  Concurrent first calls
// may both run `set`, which is harmless (it sets the same values).  Devices
// past 63 run it on every call.
template <typename F>
cudaError_t once_per_device(std::atomic<unsigned long long>& done, F set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = set();
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ---- activation rotate + quantise (rotate_quant.cu)
struct ActArgs {
  const void* x;
  qvla_dtype xdt;
  int M, ldx, K, block;
  const int32_t* perm;
  const float* rot;
  const uint16_t* rot_tc; // tensor-core image of R_B or nullptr
  int dynamic;            // 1: per-token absmax, 0: table
  const float* table;
  int T, Lcount;
  const int32_t* step_dev;
  int step_host, layer;
  uint8_t* xq;
  float* s_x;
  float* xr_out;          // rotate-only mode when non-null and xq == nullptr
  void* ws;               // optional scratch for the permuted copy of x
  size_t ws_bytes;
  int8_t* xq8;            // optional int8 image of the codes (GEMM operand order)
};
cudaError_t launch_rotate_quant(const ActArgs& a, cudaStream_t stream);
// independent linears in as few launches as possible (grouped by kernel config)
cudaError_t launch_rotate_quant_batch(const ActArgs* as, int n, cudaStream_t stream);

// quantise already-rotated fp32 rows: activations (qmin -8) or weights (qmin -7)
struct QuantArgs {
  const float* xr;
  int rows, K;
  int qmin, qmax;
  int dynamic;
  const float* table;
  int T, Lcount;
  const int32_t* step_dev;
  int step_host, layer;
  uint8_t* q_out;          // [rows][K/2] packed 4-bit codes, or [rows][K] int8 when bits == 8
  float* s_out;
  int bits;                // 4 (default when 0) or 8
};
cudaError_t launch_quant_rows(const QuantArgs& a, cudaStream_t stream);
// independent row sets in as few launches as possible (one CTA per row)
cudaError_t launch_quant_rows_batch(const QuantArgs* as, int n, cudaStream_t stream);

// ---- GPTQ rounding on the host (gptq_host.cu)
// H = X'^T X' (fp64, K x K) of T rotated calibration rows xr [T][K].
void gptq_hessian(const float* xr, int T, int K, std::vector<double>& H);
// U = upper Cholesky factor of (H + damp * mean(diag H) * I)^-1 after giving
// dead inputs (H[i][i] == 0, flagged in `dead`) a unit diagonal; false if a
// factorisation fails.
bool gptq_inverse_factor(const double* H, int K, double damp, std::vector<double>& U,
                         std::vector<char>& dead);
// codes [N][K] (one int8 each) and fp32 scales [N] of fp32 rotated weights;
// `dead` may be null.
void gptq_quantize_rows(const float* Wr, int N, int K, const double* U, const char* dead, int qmax,
                        int8_t* q, float* s);

// ---- pack helpers (pack_kernels.cu)
cudaError_t launch_column_norms(const float* W, int N, int K, double* norms, cudaStream_t s);
cudaError_t launch_block_gram(const float* W, int N, int K, int block, const int32_t* perm,
                              double* gram, cudaStream_t s);
cudaError_t launch_rot_tc_image(const double* rsvd64, int K, int block, uint16_t* img,
                                cudaStream_t s);
cudaError_t launch_rotate_weights(const float* W, int N, int K, int block, const int32_t* perm,
                                  const double* rsvd64, float* Wr, cudaStream_t s);

// ---- GEMM (gemm_w4a4.cu)
struct GemmArgs {
  const uint8_t* xq;
  const int8_t* xq8;      // int8 image of the codes, or nullptr (unpack xq)
  const float* s_x;
  int M, N, K;
  const uint8_t* wq;
  const float* w_scale;
  const float* bias;
  void* y;                // bf16 [M][ldy] or nullptr
  int ldy;
  int32_t* acc;           // int32 [M][N] when y == nullptr
  int split_k;
};
cudaError_t launch_w4a4_gemm(const GemmArgs& g, cudaStream_t stream);

// 2-D tiled tensor map over a row-major array (`inner` elements per row,
// `outer` rows, row pitch `pitch` bytes), box `box_inner` x `box_outer`.
bool encode_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t inner,
                   uint64_t outer, uint64_t pitch, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle);
// independent linears in as few launches as possible (grouped by token tile)
cudaError_t launch_w4a4_gemm_batch(const GemmArgs* gs, int n, int split_k, cudaStream_t stream);
// W8A8 variant (gemm_w8a8.cu): int8 codes [M][K] and [N][K] straight into the
// tensor cores (xq and wq hold one int8 code per byte; split_k is ignored)
cudaError_t launch_w8a8_gemm(const GemmArgs& g, cudaStream_t stream);
// independent W8A8 linears, grouped by token tile, up to 16 per launch
cudaError_t launch_w8a8_gemm_batch(const GemmArgs* gs, int n, cudaStream_t stream);

}  // namespace qvla
