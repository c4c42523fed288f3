// abi_check.cpp -- a C++ client of the library's C ABI.
//
// Compiled against include/bitlinear.h and linked to libbitlinear.so by
// tests/test_abi_cpp.py.  Without arguments it runs the host-side checks
// (sizes, argument validation, status strings: no GPU needed); with --gpu it
// also packs host-made ternary codes, runs the forward on int8 tokens with
// INT32 output (one decode-sized and one tensor-core-sized case) and compares
// every accumulator with a brute-force sum computed here on the host.
// Exit status 0 when every check holds.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <vector>

#include "bitlinear.h"

static int g_fails = 0;
#define CHECK(c)                                                              \
  do {                                                                        \
    if (!(c)) {                                                               \
      std::fprintf(stderr, "FAIL %s:%d: %s\n", __FILE__, __LINE__, #c);      \
      ++g_fails;                                                              \
    }                                                                         \
  } while (0)

static void host_checks() {
  // packed row strides: ceil(K / per) rounded up to 16 bytes
  CHECK(bitlinear_packed_row_bytes(3200, BL_PACK_I2) == 800);
  CHECK(bitlinear_packed_row_bytes(3200, BL_PACK_T5) == 640);
  CHECK(bitlinear_packed_row_bytes(3200, BL_PACK_B1) == 400);
  CHECK(bitlinear_packed_row_bytes(8640, BL_PACK_I2) == 2160);
  CHECK(bitlinear_packed_row_bytes(1, BL_PACK_I2) == 16);
  CHECK(bitlinear_packed_row_bytes(0, BL_PACK_I2) == -1);
  CHECK(bitlinear_packed_row_bytes(5, 9) == -1);
  // workspace sizes: at least the header when valid, 0 when not
  CHECK(bitlinear_quantize_weights_workspace_bytes(512, 256) == BL_WS_HEADER_BYTES + 256);
  CHECK(bitlinear_quantize_weights_workspace_bytes(0, 256) == 0);
  CHECK(bitlinear_forward_workspace_bytes(1, 8640, 3200, BL_PACK_I2, BL_BF16) >= BL_WS_HEADER_BYTES);
  CHECK(bitlinear_forward_workspace_bytes(1, 8640, 0, BL_PACK_I2, BL_BF16) == 0);
  CHECK(bitlinear_binarize_weights_workspace_bytes(512, 256) == BL_WS_HEADER_BYTES + 256);
  const int64_t rows[3] = {3200, 3200, 3200};
  CHECK(bitlinear_forward_grouped_workspace_bytes(1, 3, rows, 3200, BL_PACK_I2, BL_BF16) == BL_WS_HEADER_BYTES);
  CHECK(bitlinear_forward_grouped_workspace_bytes(1, 9, rows, 3200, BL_PACK_I2, BL_BF16) == 0);
  CHECK(bitlinear_backward_dx_workspace_bytes(1, 512, 256, BL_PACK_I2) > BL_WS_HEADER_BYTES);

  // argument validation happens on the host, before any launch
  void* p = reinterpret_cast<void*>(uintptr_t{1} << 20);  // aligned, never dereferenced
  void* odd = reinterpret_cast<void*>((uintptr_t{1} << 20) + 4);
  const uint8_t* pk = static_cast<const uint8_t*>(p);
  float* pf = static_cast<float*>(p);
  CHECK(bitlinear_forward(nullptr, BL_PACK_I2, pf, 4, 4, p, BL_BF16, pf, 1, p, BL_BF16, p, 4096, nullptr) ==
        BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_forward(pk, 7, pf, 4, 4, p, BL_BF16, pf, 1, p, BL_BF16, p, 4096, nullptr) == BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_forward(pk, BL_PACK_I2, pf, 4, 0, p, BL_BF16, pf, 1, p, BL_BF16, p, 4096, nullptr) ==
        BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_forward(pk, BL_PACK_I2, pf, 4, 4, odd, BL_BF16, pf, 1, p, BL_BF16, p, 4096, nullptr) ==
        BL_ERR_MISALIGNED);
  CHECK(bitlinear_forward(pk, BL_PACK_I2, pf, 4, 4, p, BL_BF16, pf, 1, p, BL_BF16, p, 8, nullptr) ==
        BL_ERR_WORKSPACE_TOO_SMALL);
  CHECK(bitlinear_forward(pk, BL_PACK_I2, pf, 4, 4, p, BL_BF16, pf, 0, p, BL_BF16, p, 4096, nullptr) == BL_OK);
  CHECK(bitlinear_quantize_weights(p, BL_F32, 4, 4, 0.0f, BL_PACK_I2, static_cast<uint8_t*>(p), nullptr, pf, p, 4096,
                                   nullptr) == BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_quantize_weights(p, BL_F32, 4, 4, 1e-5f, BL_PACK_B1, static_cast<uint8_t*>(p), nullptr, pf, p,
                                   4096, nullptr) == BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_binarize_weights(p, BL_F32, 4, 4, nullptr, nullptr, pf, pf, p, 4096, nullptr) ==
        BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_quantize_acts(p, BL_I8, 4, 4, static_cast<int8_t*>(p), pf, nullptr) == BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_backward_dw(p, BL_F32, static_cast<const int8_t*>(p), pf, pf, 1, 4, 4, nullptr, nullptr) ==
        BL_ERR_INVALID_VALUE);
  CHECK(bitlinear_workspace_init(nullptr, 4096, nullptr) == BL_ERR_INVALID_VALUE);
  CHECK(std::strncmp(bitlinear_status_string(BL_OK), "BL_OK", 5) == 0);
  CHECK(std::strncmp(bitlinear_status_string(BL_ERR_DEVICE_TIMEOUT), "BL_ERR_DEVICE_TIMEOUT", 21) == 0);
  CHECK(bitlinear_version() >= 100);
}

// ---- GPU part (--gpu) ----------------------------------------------------------------
#include <cuda_runtime.h>

static uint32_t g_lcg = 12345u;
static uint32_t lcg() {
  g_lcg = g_lcg * 1664525u + 1013904223u;
  return g_lcg >> 8;
}

#define CUDA_OK(e) CHECK((e) == cudaSuccess)

// Pack host codes, run the forward on int8 tokens with INT32 output, compare
// with the brute-force products.
static void forward_case(int64_t M, int64_t N, int64_t K) {
  std::vector<int8_t> codes(N * K), xq(M * K);
  for (auto& c : codes) c = static_cast<int8_t>(static_cast<int>(lcg() % 3u) - 1);
  for (auto& v : xq) v = static_cast<int8_t>(static_cast<int>(lcg() % 255u) - 127);
  std::vector<float> scale(M, 1.0f);
  const float gamma = 0.5f;
  const int64_t rb = bitlinear_packed_row_bytes(K, BL_PACK_I2);
  const size_t fws = bitlinear_forward_workspace_bytes(M, N, K, BL_PACK_I2, BL_I8);
  void *d_codes = nullptr, *d_packed = nullptr, *d_x = nullptr, *d_s = nullptr, *d_g = nullptr, *d_y = nullptr,
       *d_ws = nullptr;
  CUDA_OK(cudaMalloc(&d_codes, N * K));
  CUDA_OK(cudaMalloc(&d_packed, N * rb));
  CUDA_OK(cudaMalloc(&d_x, M * K));
  CUDA_OK(cudaMalloc(&d_s, M * sizeof(float)));
  CUDA_OK(cudaMalloc(&d_g, sizeof(float)));
  CUDA_OK(cudaMalloc(&d_y, M * N * sizeof(int32_t)));
  CUDA_OK(cudaMalloc(&d_ws, fws < 4096 ? 4096 : fws));
  if (g_fails) return;
  CUDA_OK(cudaMemcpy(d_codes, codes.data(), N * K, cudaMemcpyHostToDevice));
  CUDA_OK(cudaMemcpy(d_x, xq.data(), M * K, cudaMemcpyHostToDevice));
  CUDA_OK(cudaMemcpy(d_s, scale.data(), M * sizeof(float), cudaMemcpyHostToDevice));
  CUDA_OK(cudaMemcpy(d_g, &gamma, sizeof(float), cudaMemcpyHostToDevice));
  CHECK(bitlinear_workspace_init(d_ws, fws < 4096 ? 4096 : fws, nullptr) == BL_OK);
  CHECK(bitlinear_pack(static_cast<const int8_t*>(d_codes), N, K, BL_PACK_I2, static_cast<uint8_t*>(d_packed), d_ws,
                       fws < 4096 ? 4096 : fws, nullptr) == BL_OK);
  CHECK(bitlinear_forward(static_cast<const uint8_t*>(d_packed), BL_PACK_I2, static_cast<const float*>(d_g), N, K,
                          d_x, BL_I8, static_cast<float*>(d_s), M, d_y, BL_I32, d_ws, fws < 4096 ? 4096 : fws,
                          nullptr) == BL_OK);
  CUDA_OK(cudaDeviceSynchronize());
  CHECK(bitlinear_device_status(d_ws, nullptr) == BL_OK);
  std::vector<int32_t> y(M * N, 0);
  CUDA_OK(cudaMemcpy(y.data(), d_y, M * N * sizeof(int32_t), cudaMemcpyDeviceToHost));
  int64_t bad = 0;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += int64_t{codes[n * K + k]} * int64_t{xq[m * K + k]};
      if (s != y[m * N + n]) ++bad;
    }
  if (bad) std::fprintf(stderr, "M=%lld N=%lld K=%lld: %lld accumulators differ\n", (long long)M, (long long)N,
                        (long long)K, (long long)bad);
  CHECK(bad == 0);
  cudaFree(d_codes);
  cudaFree(d_packed);
  cudaFree(d_x);
  cudaFree(d_s);
  cudaFree(d_g);
  cudaFree(d_y);
  cudaFree(d_ws);
}

int main(int argc, char** argv) {
  host_checks();
  if (argc > 1 && std::strcmp(argv[1], "--gpu") == 0) {
    forward_case(3, 37, 200);    // decode GEMV (K not a multiple of 16)
    forward_case(20, 300, 256);  // tensor-core path
  }
  std::printf("%s (%d failed checks)\n", g_fails ? "FAIL" : "OK", g_fails);
  return g_fails ? 1 : 0;
}
