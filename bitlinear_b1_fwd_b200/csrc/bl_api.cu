// bl_api.cu -- the C ABI declared in include/bitlinear.h: argument checks on the
// host, workspace carving, and kernel selection.  Nothing here computes.
#include <cmath>
#include <cstring>

#include "bitlinear.h"
#include "bl_common.cuh"
#include "bl_kernels.h"

namespace {

constexpr int64_t kMaxK = int64_t{1} << 20;
constexpr int64_t kMaxNK = int64_t{1} << 32;
// Rows of W (N) and tokens (M) stay below 2^31: the kernels count rows,
// tokens and per-row work items in 32-bit integers (with K = 1, N up to
// 2^32 would satisfy N K <= 2^32 but overflow those counts).
constexpr int64_t kMaxRows = (int64_t{1} << 31) - 1;
constexpr int kVersion = 100;  // 0.1.0

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline size_t round256(size_t v) { return (v + 255) / 256 * 256; }
inline bool float_dt(int dt) { return dt == BL_F32 || dt == BL_BF16; }
inline bool fmt_ok(int fmt) { return fmt == BL_PACK_I2 || fmt == BL_PACK_T5 || fmt == BL_PACK_B1; }
inline bool tern_fmt_ok(int fmt) { return fmt == BL_PACK_I2 || fmt == BL_PACK_T5; }  // ternary formats

inline bl_status cuda_status(cudaError_t e) { return e == cudaSuccess ? BL_OK : BL_ERR_CUDA; }

bool nk_ok(int64_t N, int64_t K) {
  if (N < 0 || N > kMaxRows || K < 1 || K > kMaxK) return false;
  return N <= kMaxNK / K;
}

inline bool m_ok(int64_t M) { return M >= 0 && M <= kMaxRows; }

}  // namespace

extern "C" {

int bitlinear_version(void) { return kVersion; }

const char* bitlinear_status_string(int status) {
  switch (status) {
    case BL_OK: return "BL_OK: success";
    case BL_ERR_INVALID_VALUE: return "BL_ERR_INVALID_VALUE: a size, dtype, format or pointer is invalid";
    case BL_ERR_UNSUPPORTED: return "BL_ERR_UNSUPPORTED: valid arguments, but not supported on this device";
    case BL_ERR_MISALIGNED: return "BL_ERR_MISALIGNED: an array pointer is not 16-byte aligned";
    case BL_ERR_WORKSPACE_TOO_SMALL: return "BL_ERR_WORKSPACE_TOO_SMALL: workspace below the queried size";
    case BL_ERR_CUDA: return "BL_ERR_CUDA: a CUDA runtime call failed";
    case BL_ERR_DEVICE_TIMEOUT: return "BL_ERR_DEVICE_TIMEOUT: a bounded wait in a kernel ran out";
    case BL_ERR_BAD_CODE: return "BL_ERR_BAD_CODE: a weight code outside {-1, 0, 1} was packed";
    case BL_ERR_SCRATCH_LIMIT:
      return "BL_ERR_SCRATCH_LIMIT: N*K exceeds the fixed scratch of bitlinear_absmean_noalloc (2^28 elements)";
    default: return "unknown bitlinear status";
  }
}

int64_t bitlinear_packed_row_bytes(int64_t K, int fmt) {
  if (K < 1 || K > kMaxK || !fmt_ok(fmt)) return -1;
  const int64_t per = fmt == BL_PACK_I2 ? 4 : (fmt == BL_PACK_T5 ? 5 : 8);
  return ((K + per - 1) / per + 15) / 16 * 16;
}

size_t bitlinear_quantize_weights_workspace_bytes(int64_t N, int64_t K) {
  if (N < 1 || !nk_ok(N, K)) return 0;
  const int64_t chunks = (N * K + bl::kChunk - 1) / bl::kChunk;
  return BL_WS_HEADER_BYTES + round256(static_cast<size_t>(chunks) * sizeof(double));
}

// The tensor-core path serves more tokens than one GEMV launch holds, when the
// x_q rows can be a TMA tensor (row stride a multiple of 16 bytes).
bool uses_gemm(int64_t M, int64_t K) { return M > bl::kGemvMaxTokens && (K % 16) == 0; }
// 1-bit rows longer than the 1-bit GEMV takes (4096 bytes: K > 32768) are
// transcoded to 2 bits in the workspace for the decode path too.
bool b1_via_i2(int fmt, int64_t K) { return fmt == BL_PACK_B1 && (K + 7) / 8 > 4096; }

size_t bitlinear_forward_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int xdt) {
  if (!m_ok(M) || !nk_ok(N, K) || !fmt_ok(fmt)) return 0;
  size_t bytes = BL_WS_HEADER_BYTES;
  if (uses_gemm(M, K)) {
    if (xdt != BL_I8) bytes += round256(static_cast<size_t>(M * K));
    if (fmt != BL_PACK_I2) bytes += round256(static_cast<size_t>(N * bitlinear_packed_row_bytes(K, BL_PACK_I2)));
    const int ks = bl::gemm_split_k(M, N, K);
    if (ks > 1) bytes += round256(static_cast<size_t>(ks) * M * N * sizeof(int32_t));
  } else if (b1_via_i2(fmt, K)) {
    bytes += round256(static_cast<size_t>(N * bitlinear_packed_row_bytes(K, BL_PACK_I2)));
  }
  return bytes;
}

bl_status bitlinear_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < BL_WS_HEADER_BYTES) return BL_ERR_INVALID_VALUE;
  return cuda_status(cudaMemsetAsync(ws, 0, BL_WS_HEADER_BYTES, static_cast<cudaStream_t>(stream)));
}

bl_status bitlinear_quantize_weights(const void* W, int wdt, int64_t N, int64_t K, float eps, int fmt,
                                     uint8_t* packed, int8_t* codes, float* gamma, void* ws,
                                     size_t ws_bytes, void* stream) {
  if (W == nullptr || gamma == nullptr || ws == nullptr || (packed == nullptr && codes == nullptr))
    return BL_ERR_INVALID_VALUE;
  if (!float_dt(wdt) || !tern_fmt_ok(fmt) || N < 1 || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (!(eps > 0.0f) || !std::isfinite(eps)) return BL_ERR_INVALID_VALUE;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(codes, 16) || !aligned(gamma, 4) ||
      !aligned(ws, 16))
    return BL_ERR_MISALIGNED;
  if (ws_bytes < bitlinear_quantize_weights_workspace_bytes(N, K)) return BL_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = bl::launch_absmean(W, wdt, N, K, ws, gamma, st);
  if (e != cudaSuccess) return BL_ERR_CUDA;
  const int64_t rb = bitlinear_packed_row_bytes(K, fmt);
  return cuda_status(bl::launch_ternarize_pack(W, wdt, N, K, gamma, eps, fmt, packed, codes, rb, ws, st));
}

bl_status bitlinear_absmean(const void* W, int wdt, int64_t N, int64_t K, float* gamma, void* ws,
                            size_t ws_bytes, void* stream) {
  if (W == nullptr || gamma == nullptr || ws == nullptr) return BL_ERR_INVALID_VALUE;
  if (!float_dt(wdt) || N < 1 || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (!aligned(W, 16) || !aligned(gamma, 4) || !aligned(ws, 16)) return BL_ERR_MISALIGNED;
  if (ws_bytes < bitlinear_quantize_weights_workspace_bytes(N, K)) return BL_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(bl::launch_absmean(W, wdt, N, K, ws, gamma, static_cast<cudaStream_t>(stream)));
}

bl_status bitlinear_ternarize_pack(const void* W, int wdt, int64_t N, int64_t K, const float* gamma,
                                   float eps, int fmt, uint8_t* packed, int8_t* codes, void* stream) {
  if (W == nullptr || gamma == nullptr || (packed == nullptr && codes == nullptr)) return BL_ERR_INVALID_VALUE;
  if (!float_dt(wdt) || !tern_fmt_ok(fmt) || N < 1 || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (!(eps > 0.0f) || !std::isfinite(eps)) return BL_ERR_INVALID_VALUE;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(codes, 16) || !aligned(gamma, 4))
    return BL_ERR_MISALIGNED;
  const int64_t rb = bitlinear_packed_row_bytes(K, fmt);
  return cuda_status(bl::launch_ternarize_pack(W, wdt, N, K, gamma, eps, fmt, packed, codes, rb, nullptr,
                                               static_cast<cudaStream_t>(stream)));
}

size_t bitlinear_binarize_weights_workspace_bytes(int64_t N, int64_t K) {
  if (N < 1 || !nk_ok(N, K)) return 0;
  const int64_t chunks = (N * K + bl::kChunk - 1) / bl::kChunk;
  return BL_WS_HEADER_BYTES + round256(static_cast<size_t>(2 * chunks) * sizeof(double));
}

bl_status bitlinear_binarize_weights(const void* W, int wdt, int64_t N, int64_t K, uint8_t* packed, int8_t* codes,
                                     float* beta, float* alpha, void* ws, size_t ws_bytes, void* stream) {
  if (W == nullptr || beta == nullptr || alpha == nullptr || ws == nullptr || (packed == nullptr && codes == nullptr))
    return BL_ERR_INVALID_VALUE;
  if (!float_dt(wdt) || N < 1 || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(codes, 16) || !aligned(beta, 4) || !aligned(alpha, 4) ||
      !aligned(ws, 16))
    return BL_ERR_MISALIGNED;
  if (ws_bytes < bitlinear_binarize_weights_workspace_bytes(N, K)) return BL_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (bl::launch_absmean(W, wdt, N, K, ws, beta, st, alpha) != cudaSuccess) return BL_ERR_CUDA;
  const int64_t rb = bitlinear_packed_row_bytes(K, BL_PACK_B1);
  return cuda_status(bl::launch_binarize_pack(W, wdt, N, K, alpha, packed, codes, rb, st));
}

bl_status bitlinear_pack(const int8_t* codes, int64_t N, int64_t K, int fmt, uint8_t* packed, void* ws,
                         size_t ws_bytes, void* stream) {
  if (!fmt_ok(fmt) || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (N == 0) return BL_OK;
  if (codes == nullptr || packed == nullptr || ws == nullptr) return BL_ERR_INVALID_VALUE;
  if (!aligned(codes, 16) || !aligned(packed, 16) || !aligned(ws, 16)) return BL_ERR_MISALIGNED;
  if (ws_bytes < BL_WS_HEADER_BYTES) return BL_ERR_WORKSPACE_TOO_SMALL;
  const int64_t rb = bitlinear_packed_row_bytes(K, fmt);
  return cuda_status(bl::launch_pack(codes, N, K, fmt, packed, rb, ws, static_cast<cudaStream_t>(stream)));
}

bl_status bitlinear_quantize_acts(const void* x, int xdt, int64_t M, int64_t K, int8_t* xq, float* scale,
                                  void* stream) {
  if (!float_dt(xdt) || !m_ok(M) || K < 1 || K > kMaxK) return BL_ERR_INVALID_VALUE;
  if (M == 0) return BL_OK;
  if (x == nullptr || xq == nullptr || scale == nullptr) return BL_ERR_INVALID_VALUE;
  if (!aligned(x, 16) || !aligned(xq, 16) || !aligned(scale, 4)) return BL_ERR_MISALIGNED;
  return cuda_status(bl::launch_act_quant(x, xdt, M, K, xq, scale, static_cast<cudaStream_t>(stream)));
}

bl_status bitlinear_layernorm_quantize_acts(const void* x, int xdt, const float* ln_w, const float* ln_b, float eps,
                                            int64_t M, int64_t K, uint16_t* y, int8_t* xq, float* scale,
                                            void* stream) {
  if (!float_dt(xdt) || !m_ok(M) || K < 1 || K > kMaxK) return BL_ERR_INVALID_VALUE;
  if (!(eps > 0.0f) || !std::isfinite(eps)) return BL_ERR_INVALID_VALUE;
  if (M == 0) return BL_OK;
  if (x == nullptr || ln_w == nullptr || ln_b == nullptr || xq == nullptr || scale == nullptr)
    return BL_ERR_INVALID_VALUE;
  if (!aligned(x, 16) || !aligned(ln_w, 4) || !aligned(ln_b, 4) || !aligned(y, 2) || !aligned(scale, 4))
    return BL_ERR_MISALIGNED;
  return cuda_status(bl::launch_ln_quant(x, xdt, ln_w, ln_b, eps, M, K, y, xq, scale, static_cast<cudaStream_t>(stream)));
}

bl_status bitlinear_forward(const uint8_t* packed, int fmt, const float* gamma, int64_t N, int64_t K,
                            const void* x, int xdt, float* scale, int64_t M, void* y, int ydt, void* ws,
                            size_t ws_bytes, void* stream) {
  if (!fmt_ok(fmt) || !(float_dt(xdt) || xdt == BL_I8) || !(float_dt(ydt) || ydt == BL_I32))
    return BL_ERR_INVALID_VALUE;
  if (!m_ok(M) || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (M == 0 || N == 0) return BL_OK;  // empty output: nothing to read or write
  if (packed == nullptr || gamma == nullptr || x == nullptr || scale == nullptr || y == nullptr ||
      ws == nullptr)
    return BL_ERR_INVALID_VALUE;
  if (!aligned(packed, 16) || !aligned(x, 16) || !aligned(y, 16) || !aligned(scale, 4) ||
      !aligned(gamma, 4) || !aligned(ws, 16))
    return BL_ERR_MISALIGNED;
  if (ws_bytes < bitlinear_forward_workspace_bytes(M, N, K, fmt, xdt)) return BL_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!uses_gemm(M, K)) {
    if (b1_via_i2(fmt, K)) {
      uint8_t* w2 = static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES;
      const int64_t rb2 = bitlinear_packed_row_bytes(K, BL_PACK_I2);
      if (bl::launch_b1_to_i2(packed, N, K, bitlinear_packed_row_bytes(K, fmt), w2, rb2, st) != cudaSuccess)
        return BL_ERR_CUDA;
      packed = w2;
      fmt = BL_PACK_I2;
    }
    if (bl::gemv_max_tokens(fmt, bitlinear_packed_row_bytes(K, fmt)) < 1) return BL_ERR_UNSUPPORTED;
    return cuda_status(bl::launch_gemv(packed, fmt, gamma, N, K, x, xdt, scale, M, y, ydt, bl::one_group(N), ws, st));
  }
  uint8_t* scratch = static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES;
  const int8_t* xq = static_cast<const int8_t*>(x);
  if (xdt != BL_I8) {
    if (bl::launch_act_quant(x, xdt, M, K, reinterpret_cast<int8_t*>(scratch), scale, st) != cudaSuccess)
      return BL_ERR_CUDA;
    xq = reinterpret_cast<const int8_t*>(scratch);
    scratch += round256(static_cast<size_t>(M * K));
  }
  const int64_t rb2 = bitlinear_packed_row_bytes(K, BL_PACK_I2);
  const uint8_t* w2 = packed;
  if (fmt != BL_PACK_I2) {
    const int64_t rb = bitlinear_packed_row_bytes(K, fmt);
    const cudaError_t e = fmt == BL_PACK_T5 ? bl::launch_t5_to_i2(packed, N, K, rb, scratch, rb2, st)
                                            : bl::launch_b1_to_i2(packed, N, K, rb, scratch, rb2, st);
    if (e != cudaSuccess) return BL_ERR_CUDA;
    w2 = scratch;
    scratch += round256(static_cast<size_t>(N * rb2));
  }
  int32_t* part = bl::gemm_split_k(M, N, K) > 1 ? reinterpret_cast<int32_t*>(scratch) : nullptr;
  return cuda_status(bl::launch_gemm_i2(xq, w2, rb2, gamma, scale, y, ydt, M, N, K, N, part, ws, 0, 0, st));
}

// Several weight matrices sharing one token batch (for example a block's Q, K
// and V projections): their packed rows are concatenated, each group has its
// own gamma, and y holds the groups' outputs side by side.
static int64_t group_total(int64_t ngroups, const int64_t* group_rows) {
  if (ngroups < 1 || ngroups > bl::kMaxRowGroups || group_rows == nullptr) return -1;
  int64_t n = 0;
  for (int64_t g = 0; g < ngroups; ++g) {
    if (group_rows[g] < 1) return -1;
    n += group_rows[g];
  }
  return n;
}

size_t bitlinear_forward_grouped_workspace_bytes(int64_t M, int64_t ngroups, const int64_t* group_rows, int64_t K,
                                                 int fmt, int xdt) {
  const int64_t N = group_total(ngroups, group_rows);
  if (N < 1 || !m_ok(M) || !nk_ok(N, K) || !fmt_ok(fmt)) return 0;
  size_t bytes = BL_WS_HEADER_BYTES;
  if (uses_gemm(M, K)) {
    if (xdt != BL_I8) bytes += round256(static_cast<size_t>(M * K));
    size_t most = 0;  // the groups run one after another and share the rest
    for (int64_t g = 0; g < ngroups; ++g) {
      const int64_t Ng = group_rows[g];
      size_t e = 0;
      if (fmt != BL_PACK_I2) e += round256(static_cast<size_t>(Ng * bitlinear_packed_row_bytes(K, BL_PACK_I2)));
      const int ks = bl::gemm_split_k(M, Ng, K);
      if (ks > 1) e += round256(static_cast<size_t>(ks) * M * Ng * sizeof(int32_t));
      if (e > most) most = e;
    }
    bytes += most;
  } else if (b1_via_i2(fmt, K)) {
    bytes += round256(static_cast<size_t>(N * bitlinear_packed_row_bytes(K, BL_PACK_I2)));
  }
  return bytes;
}

bl_status bitlinear_forward_grouped(const uint8_t* packed, int fmt, const float* gammas, int64_t ngroups,
                                    const int64_t* group_rows, int64_t K, const void* x, int xdt, float* scale,
                                    int64_t M, void* y, int ydt, void* ws, size_t ws_bytes, void* stream) {
  if (!fmt_ok(fmt) || !(float_dt(xdt) || xdt == BL_I8) || !(float_dt(ydt) || ydt == BL_I32))
    return BL_ERR_INVALID_VALUE;
  const int64_t N = group_total(ngroups, group_rows);
  if (N < 1 || !m_ok(M) || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (M == 0) return BL_OK;
  if (packed == nullptr || gammas == nullptr || x == nullptr || scale == nullptr || y == nullptr || ws == nullptr)
    return BL_ERR_INVALID_VALUE;
  if (!aligned(packed, 16) || !aligned(x, 16) || !aligned(y, 16) || !aligned(scale, 4) || !aligned(gammas, 4) ||
      !aligned(ws, 16))
    return BL_ERR_MISALIGNED;
  if (ws_bytes < bitlinear_forward_grouped_workspace_bytes(M, ngroups, group_rows, K, fmt, xdt))
    return BL_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rb = bitlinear_packed_row_bytes(K, fmt);
  if (!uses_gemm(M, K)) {  // one GEMV launch over every group's rows
    if (b1_via_i2(fmt, K)) {
      uint8_t* w2 = static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES;
      if (bl::launch_b1_to_i2(packed, N, K, rb, w2, bitlinear_packed_row_bytes(K, BL_PACK_I2), st) != cudaSuccess)
        return BL_ERR_CUDA;
      packed = w2;
      fmt = BL_PACK_I2;
    }
    if (bl::gemv_max_tokens(fmt, bitlinear_packed_row_bytes(K, fmt)) < 1) return BL_ERR_UNSUPPORTED;
    bl::RowGroups rg{};
    rg.n = static_cast<int>(ngroups);
    int64_t end = 0;
    for (int64_t g = 0; g < ngroups; ++g) rg.end[g] = (end += group_rows[g]);
    return cuda_status(bl::launch_gemv(packed, fmt, gammas, N, K, x, xdt, scale, M, y, ydt, rg, ws, st));
  }
  // one activation quantization, then each group's product into its columns of y
  uint8_t* scratch = static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES;
  const int8_t* xq = static_cast<const int8_t*>(x);
  if (xdt != BL_I8) {
    if (bl::launch_act_quant(x, xdt, M, K, reinterpret_cast<int8_t*>(scratch), scale, st) != cudaSuccess)
      return BL_ERR_CUDA;
    xq = reinterpret_cast<const int8_t*>(scratch);
    scratch += round256(static_cast<size_t>(M * K));
  }
  const int64_t rb2 = bitlinear_packed_row_bytes(K, BL_PACK_I2);
  const size_t ysize = (ydt == BL_BF16) ? 2 : 4;
  int64_t off = 0;
  for (int64_t g = 0; g < ngroups; ++g) {
    const int64_t Ng = group_rows[g];
    uint8_t* s2 = scratch;
    const uint8_t* w2 = packed + off * rb;
    if (fmt != BL_PACK_I2) {
      const cudaError_t ce = fmt == BL_PACK_T5 ? bl::launch_t5_to_i2(w2, Ng, K, rb, s2, rb2, st)
                                               : bl::launch_b1_to_i2(w2, Ng, K, rb, s2, rb2, st);
      if (ce != cudaSuccess) return BL_ERR_CUDA;
      w2 = s2;
      s2 += round256(static_cast<size_t>(Ng * rb2));
    }
    int32_t* part = bl::gemm_split_k(M, Ng, K) > 1 ? reinterpret_cast<int32_t*>(s2) : nullptr;
    const bl_status e = cuda_status(bl::launch_gemm_i2(xq, w2, rb2, gammas + g, scale, static_cast<uint8_t*>(y) + off * ysize,
                                                       ydt, M, Ng, K, N, part, ws, 0, 0, st));
    if (e != BL_OK) return e;
    off += Ng;
  }
  return BL_OK;
}

// STE backward.
size_t bitlinear_backward_dx_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt) {
  if (N < 1 || !m_ok(M) || !nk_ok(N, K) || !fmt_ok(fmt)) return 0;
  size_t bytes = BL_WS_HEADER_BYTES;
  if (fmt != BL_PACK_I2) bytes += round256(static_cast<size_t>(N * bitlinear_packed_row_bytes(K, BL_PACK_I2)));
  const int64_t mt = M < bl::backward_dx_tokens_per_pass() ? M : bl::backward_dx_tokens_per_pass();
  bytes += round256(static_cast<size_t>(bl::backward_dx_chunks(N) * mt * K) * sizeof(double));
  return bytes;
}

bl_status bitlinear_backward_dx(const uint8_t* packed, int fmt, const float* gamma, int64_t N, int64_t K,
                                const void* dy, int dydt, int64_t M, float* dx, void* ws, size_t ws_bytes,
                                void* stream) {
  if (!fmt_ok(fmt) || !float_dt(dydt) || !m_ok(M) || N < 1 || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (M == 0) return BL_OK;
  if (packed == nullptr || gamma == nullptr || dy == nullptr || dx == nullptr || ws == nullptr)
    return BL_ERR_INVALID_VALUE;
  if (!aligned(packed, 16) || !aligned(dy, 16) || !aligned(dx, 16) || !aligned(gamma, 4) || !aligned(ws, 16))
    return BL_ERR_MISALIGNED;
  if (ws_bytes < bitlinear_backward_dx_workspace_bytes(M, N, K, fmt)) return BL_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* scratch = static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES;
  const int64_t rb2 = bitlinear_packed_row_bytes(K, BL_PACK_I2);
  const uint8_t* w2 = packed;
  if (fmt != BL_PACK_I2) {
    const int64_t rb = bitlinear_packed_row_bytes(K, fmt);
    const cudaError_t e = fmt == BL_PACK_T5 ? bl::launch_t5_to_i2(packed, N, K, rb, scratch, rb2, st)
                                            : bl::launch_b1_to_i2(packed, N, K, rb, scratch, rb2, st);
    if (e != cudaSuccess) return BL_ERR_CUDA;
    w2 = scratch;
    scratch += round256(static_cast<size_t>(N * rb2));
  }
  return cuda_status(bl::launch_backward_dx(w2, rb2, gamma, N, K, dy, dydt, M, dx, reinterpret_cast<double*>(scratch), st));
}

bl_status bitlinear_backward_dw(const void* dy, int dydt, const int8_t* xq, const float* scale, const float* gamma,
                                int64_t M, int64_t N, int64_t K, float* dw, void* stream) {
  if (!float_dt(dydt) || !m_ok(M) || N < 1 || !nk_ok(N, K)) return BL_ERR_INVALID_VALUE;
  if (dw == nullptr || gamma == nullptr || (M > 0 && (dy == nullptr || xq == nullptr || scale == nullptr)))
    return BL_ERR_INVALID_VALUE;
  if (!aligned(dy, 16) || !aligned(xq, 16) || !aligned(dw, 16) || !aligned(scale, 4) || !aligned(gamma, 4))
    return BL_ERR_MISALIGNED;
  return cuda_status(bl::launch_backward_dw(dy, dydt, xq, scale, gamma, M, N, K, dw, static_cast<cudaStream_t>(stream)));
}

bl_status bitlinear_selftest_wait_timeout(void* ws, size_t ws_bytes, void* stream) {
  // 16 tokens x 128 rows x 128 K: the header plus 8 KB of operand space that is never touched
  if (ws == nullptr || ws_bytes < BL_WS_HEADER_BYTES + 8192) return BL_ERR_INVALID_VALUE;
  if (!aligned(ws, 16)) return BL_ERR_MISALIGNED;
  uint8_t* op = static_cast<uint8_t*>(ws) + BL_WS_HEADER_BYTES;
  const float* g = reinterpret_cast<const float*>(op);
  return cuda_status(bl::launch_gemm_i2(reinterpret_cast<const int8_t*>(op), op, 32, g, g, op, BL_I32, 16, 128,
                                        128, 128, nullptr, ws, int64_t{1} << 20, 1, static_cast<cudaStream_t>(stream)));
}

bl_status bitlinear_device_status(void* ws, void* stream) {
  if (ws == nullptr) return BL_ERR_INVALID_VALUE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  if (cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess) return BL_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BL_ERR_CUDA;
  if (h[0] != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof h, st) != cudaSuccess) return BL_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BL_ERR_CUDA;
  }
  if (h[0] & bl::kFlagTimeout) return BL_ERR_DEVICE_TIMEOUT;
  if (h[0] & bl::kFlagBadCode) return BL_ERR_BAD_CODE;
  return BL_OK;
}

}  // extern "C"
