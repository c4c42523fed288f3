// bl_kernels.h -- launchers of the BitLinear kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bl {

// Launch with programmatic stream serialization (see pdl_enter): the kernel
// may be scheduled while the previous kernel in the stream finishes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// absmean: the last CTA folds 2^lgR chunk sums per lane (lgR <= 11 allows
// 2^19 chunks of 8192 elements, so N*K <= 2^32).
constexpr int kFinishMaxLevels = 11;

// Number of SMs of the current device (cached per device).
constexpr int kMaxDevices = 64;
int device_sms();

// decode GEMV: shared memory for activations, tokens per launch.
constexpr int64_t kGemvSmemBudget = 200 * 1024;
constexpr int kGemvMaxTokens = 4;

// ws: a workspace whose header ticket is zero; partial sums follow the header.
// alpha: when given, the mean of the weights in the same order (the 1-bit
// variant; then the partial sums take 2 C doubles).
cudaError_t launch_absmean(const void* W, int wdt, int64_t N, int64_t K, void* ws, float* gamma,
                           cudaStream_t st, float* alpha = nullptr);
cudaError_t launch_binarize_pack(const void* W, int wdt, int64_t N, int64_t K, const float* alpha, uint8_t* packed,
                                 int8_t* codes, int64_t rowbytes, cudaStream_t st);
cudaError_t launch_b1_to_i2(const uint8_t* b1, int64_t N, int64_t K, int64_t rb1, uint8_t* i2, int64_t rb2,
                            cudaStream_t st);
// ws: a workspace header for device flags, or nullptr (then a bounded wait
// that runs out goes unreported).
cudaError_t launch_ternarize_pack(const void* W, int wdt, int64_t N, int64_t K, const float* gamma,
                                  float eps, int fmt, uint8_t* packed, int8_t* codes, int64_t rowbytes, void* ws,
                                  cudaStream_t st);
cudaError_t launch_pack(const int8_t* codes, int64_t N, int64_t K, int fmt, uint8_t* packed,
                        int64_t rowbytes, void* ws, cudaStream_t st);
cudaError_t launch_ln_quant(const void* x, int xdt, const float* g, const float* b, float eps, int64_t M, int64_t K,
                            uint16_t* y, int8_t* xq, float* scale, cudaStream_t st);
cudaError_t launch_act_quant(const void* x, int xdt, int64_t M, int64_t K, int8_t* xq, float* scale,
                             cudaStream_t st);
int gemv_max_tokens(int fmt, int64_t rowbytes);
// tcgen05 GEMM on 2-bit weights; limit_cycles <= 0 uses the default wait limit.
int gemm_token_tile(int64_t M);
// y: row t of the output at y + t ldy (ldy >= N).  part: ks x M x N INT32
// partial sums for the split-K one-SM path (ks = gemm_split_k(M, N, K)), or
// nullptr to keep every tile whole.
cudaError_t launch_gemm_i2(const int8_t* xq, const uint8_t* w, int64_t rb, const float* gamma, const float* scale,
                           void* y, int ydt, int64_t M, int64_t N, int64_t K, int64_t ldy, int32_t* part, void* ws,
                           long long limit_cycles, int skip_producer, cudaStream_t st);
int gemm_split_k(int64_t M, int64_t N, int64_t K);
cudaError_t launch_t5_to_i2(const uint8_t* t5, int64_t N, int64_t K, int64_t rb5, uint8_t* i2, int64_t rb2,
                            cudaStream_t st);
// Output rows in up to kMaxRowGroups consecutive groups, each with its own
// gamma (row n belongs to the first group g with n < end[g]).
constexpr int kMaxRowGroups = 8;
struct RowGroups {
  int n;
  int64_t end[kMaxRowGroups];
};
__host__ __device__ inline int row_group(const RowGroups& rg, int64_t row) {
  int g = 0;
  while (g + 1 < rg.n && row >= rg.end[g]) ++g;
  return g;
}
inline RowGroups one_group(int64_t N) {
  RowGroups rg{};
  rg.n = 1;
  rg.end[0] = N;
  return rg;
}

// STE backward: dx through fp64 partial sums part [chunks][2][K] (chunks =
// backward_dx_chunks(N)); dW straight into dw [N, K].
int64_t backward_dx_chunks(int64_t N);
int backward_dx_tokens_per_pass();
cudaError_t launch_backward_dx(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                               const void* dy, int dydt, int64_t M, float* dx, double* part, cudaStream_t st);
cudaError_t launch_backward_dw(const void* dy, int dydt, const int8_t* xq, const float* scale, const float* gamma,
                               int64_t M, int64_t N, int64_t K, float* dw, cudaStream_t st);

// One-token 2-bit GEMV (column-stationary, early start): K % 16 == 0, rows of
// at most 8192 bytes, and fp32 tokens only when K is small enough for the raw
// token words of a thread to fit (see gemv1_fits).
bool gemv1_fits(int64_t N, int64_t K, int64_t rowbytes, int xdt);
// ws: a workspace header for the device flags (a bounded wait that runs out).
cudaError_t launch_gemv1(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                         const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg, void* ws,
                         cudaStream_t st);
// The same for one token on base-3 rows (80 weights per 16-byte segment,
// digits decoded by a per-lane shared table): K % 16 == 0 and the table,
// token, ring and row sums within the two-CTAs-per-SM budget.
bool gemv1_t5_fits(int64_t N, int64_t K, int64_t rowbytes, int xdt);
cudaError_t launch_gemv1_t5(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                            const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg, void* ws,
                            cudaStream_t st);
// And on 1-bit rows (128 weights per 16-byte segment, the codes of a column
// in registers in bit-plane order), within the same budget.
bool gemv1_b1_fits(int64_t N, int64_t K, int64_t rowbytes, int xdt);
cudaError_t launch_gemv1_b1(const uint8_t* packed, int64_t rowbytes, const float* gamma, int64_t N, int64_t K,
                            const void* x, int xdt, float* scale, void* y, int ydt, const RowGroups& rg, void* ws,
                            cudaStream_t st);

cudaError_t launch_gemv(const uint8_t* packed, int fmt, const float* gamma, int64_t N, int64_t K,
                        const void* x, int xdt, float* scale, int64_t M, void* y, int ydt,
                        const RowGroups& rg, void* ws, cudaStream_t st);

}  // namespace bl
