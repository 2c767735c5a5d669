// C ABI of the library: argument validation on the host, then one kernel launch per call.
// Declarations, argument meaning, layouts and error behaviour are in include/puro_fp8.h.

#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/puro_fp8.h"
#include "host_cache.h"
#include "quant.h"

namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The kernels walk their tiles with 32-bit indices (tile + grid stays below 2^31).
bool tiles_fit(int64_t rows, int64_t row_tile, int64_t cols, int64_t col_tile) {
  const int64_t tr = (rows + row_tile - 1) / row_tile, tc = (cols + col_tile - 1) / col_tile;
  return tr <= ((1ll << 31) - (1ll << 16)) / tc;
}

// The kernels are built for sm_100a only: refuse any other device up front.
// (The answer is cached per device.)
int check_device() {
  static puro::PerDevice<int> verdict;
  int v = PURO_ERR_CUDA;
  if (!verdict.get(v, [](int dev, int &out) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
          return false;
        out = (major == 10 && minor == 0) ? PURO_OK : PURO_ERR_DEVICE;
        return true;
      }))
    return PURO_ERR_CUDA;
  return v;
}

// Argument checks of the quantisers (both scale modes); `sa` is the scales' alignment.
int check_rows(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, const uint8_t *Xq, int64_t ldq,
               const void *S, uintptr_t sa) {
  if (X == nullptr || Xq == nullptr || S == nullptr) return PURO_ERR_NULL;
  if (R < 1 || C < 128 || C % 128 != 0 || ldx < C || ldq < C) return PURO_ERR_SHAPE;
  if (R > (1ll << 31) - 1 || C / 128 > 65535 || !tiles_fit(R, 128, C, 128)) return PURO_ERR_SHAPE;
  if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(S, sa) || ldx % 8 != 0 || ldq % 16 != 0)
    return PURO_ERR_ALIGN;
  return check_device();
}

int check_cols(const uint16_t *X, int64_t T, int64_t C, int64_t ldx, const uint8_t *XqT, const void *ST,
               const uint8_t *Xq, const void *S, uintptr_t sa) {
  if (X == nullptr || XqT == nullptr || ST == nullptr) return PURO_ERR_NULL;
  if ((Xq == nullptr) != (S == nullptr)) return PURO_ERR_NULL;
  if (T < 128 || T % 128 != 0 || C < 8 || C % 8 != 0 || ldx < C) return PURO_ERR_SHAPE;
  if (Xq != nullptr && C % 128 != 0) return PURO_ERR_SHAPE;
  if (T / 128 > 65535 || (C + 127) / 128 > (1ll << 31) - 1 || !tiles_fit(T, 128, C, 128))
    return PURO_ERR_SHAPE;
  if (!aligned(X, 16) || !aligned(XqT, 16) || !aligned(ST, sa) || ldx % 8 != 0) return PURO_ERR_ALIGN;
  if (Xq != nullptr && (!aligned(Xq, 16) || !aligned(S, sa))) return PURO_ERR_ALIGN;
  return check_device();
}

int check_weight(const uint16_t *W, int64_t R, int64_t C, int64_t ldw, const uint8_t *Wq,
                 const uint8_t *WqT, const void *S, uintptr_t sa, bool device = true) {
  if (W == nullptr || Wq == nullptr || S == nullptr) return PURO_ERR_NULL;
  if (R < 1 || C < 128 || C % 128 != 0 || ldw < C) return PURO_ERR_SHAPE;
  if ((R + 127) / 128 > 65535 || C / 128 > (1ll << 31) - 1 || !tiles_fit(R, 128, C, 128))
    return PURO_ERR_SHAPE;
  if (WqT != nullptr && R % 16 != 0) return PURO_ERR_SHAPE;
  if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(S, sa) || ldw % 8 != 0) return PURO_ERR_ALIGN;
  if (WqT != nullptr && !aligned(WqT, 16)) return PURO_ERR_ALIGN;
  return device ? check_device() : PURO_OK;
}

// The checks of one GEMM's arguments (every layout); PURO_OK or the status to return.
int check_gemm(const uint8_t *Aq, const float *As, const uint8_t *Bq, const float *Bs, const void *C,
               int64_t M, int64_t N, int64_t K, int layout) {
  if (Aq == nullptr || As == nullptr || Bq == nullptr || Bs == nullptr || C == nullptr)
    return PURO_ERR_NULL;
  if (layout != PURO_FPROP && layout != PURO_DGRAD && layout != PURO_WGRAD)
    return PURO_ERR_LAYOUT;
  if (M < 1 || N < 8 || N % 8 != 0 || K < 128 || K % 128 != 0) return PURO_ERR_SHAPE;
  // 32-bit tensor-map coordinates and kernel indices
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31) - 256) return PURO_ERR_SHAPE;
  if (!tiles_fit(M, 128, N, 256)) return PURO_ERR_SHAPE;
  if (!aligned(Aq, 16) || !aligned(Bq, 16) || !aligned(C, 16) || !aligned(As, 4) ||
      !aligned(Bs, 4))
    return PURO_ERR_ALIGN;
  return PURO_OK;
}

}  // namespace

extern "C" {

int puro_fp8_quantize_1x128(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                            int64_t ldq, float *S, puro_stream_t stream) {
  if (int e = check_rows(X, R, C, ldx, Xq, ldq, S, 4)) return e;
  return puro::launch_quant_rows(X, R, C, ldx, Xq, ldq, S, stream);
}

int puro_fp8_quantize_1x128_pow2(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                                 int64_t ldq, uint8_t *S, puro_stream_t stream) {
  if (int e = check_rows(X, R, C, ldx, Xq, ldq, S, 1)) return e;
  return puro::launch_quant_rows(X, R, C, ldx, Xq, ldq, nullptr, stream, S);
}

int puro_fp8_quantize_1x128_transposed(const uint16_t *X, int64_t T, int64_t C, int64_t ldx,
                                       uint8_t *XqT, float *ST, uint8_t *Xq, float *S,
                                       puro_stream_t stream) {
  if (int e = check_cols(X, T, C, ldx, XqT, ST, Xq, S, 4)) return e;
  return puro::launch_quant_cols(X, T, C, ldx, XqT, ST, Xq, S, stream);
}

int puro_fp8_quantize_1x128_transposed_pow2(const uint16_t *X, int64_t T, int64_t C, int64_t ldx,
                                            uint8_t *XqT, uint8_t *ST, uint8_t *Xq, uint8_t *S,
                                            puro_stream_t stream) {
  if (int e = check_cols(X, T, C, ldx, XqT, ST, Xq, S, 1)) return e;
  return puro::launch_quant_cols(X, T, C, ldx, XqT, nullptr, Xq, nullptr, stream, ST, S);
}

int puro_fp8_quantize_128x128(const uint16_t *W, int64_t R, int64_t C, int64_t ldw, uint8_t *Wq,
                              uint8_t *WqT, float *S, puro_stream_t stream) {
  if (int e = check_weight(W, R, C, ldw, Wq, WqT, S, 4)) return e;
  return puro::launch_quant_weight(W, R, C, ldw, Wq, WqT, S, stream);
}

int puro_fp8_quantize_128x128_grouped(const puro_weight_problem *problems, int count, puro_stream_t stream) {
  if (problems == nullptr) return PURO_ERR_NULL;
  if (count < 1) return PURO_ERR_SHAPE;
  int64_t tiles = 0;  // the joint tile numbering of a launch is 32-bit
  for (int p = 0; p < count; ++p) {
    const puro_weight_problem &w = problems[p];
    if (int e = check_weight(w.W, w.R, w.C, w.ldw, w.Wq, w.WqT, w.S, 4, false)) return e;
    tiles += ((w.R + 127) / 128) * (w.C / 128);
    if (tiles > (1ll << 31) - 1) return PURO_ERR_SHAPE;
  }
  if (int d = check_device()) return d;
  return puro::launch_quant_weight_grouped(problems, count, stream);
}

int puro_fp8_quantize_128x128_pow2(const uint16_t *W, int64_t R, int64_t C, int64_t ldw, uint8_t *Wq,
                                   uint8_t *WqT, uint8_t *S, puro_stream_t stream) {
  if (int e = check_weight(W, R, C, ldw, Wq, WqT, S, 1)) return e;
  return puro::launch_quant_weight(W, R, C, ldw, Wq, WqT, nullptr, stream, S);
}

int puro_fp8_gemm_blockwise(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                            const float *Bs, uint16_t *C, int64_t M, int64_t N, int64_t K,
                            int layout, void *workspace, size_t ws_bytes, puro_stream_t stream) {
  (void)workspace;
  (void)ws_bytes;
  if (int e = check_gemm(Aq, As, Bq, Bs, C, M, N, K, layout)) return e;
  if (int d = check_device()) return d;
  return puro::launch_gemm_blockwise(Aq, As, Bq, Bs, C, M, N, K, layout, stream);
}

int puro_fp8_mx_gemm(const uint8_t *Aq, const uint8_t *As, const uint8_t *Bq, const uint8_t *Bs,
                     uint16_t *C, int64_t M, int64_t N, int64_t K, int layout, puro_stream_t stream) {
  if (Aq == nullptr || As == nullptr || Bq == nullptr || Bs == nullptr || C == nullptr)
    return PURO_ERR_NULL;
  if (layout != PURO_FPROP && layout != PURO_DGRAD && layout != PURO_WGRAD) return PURO_ERR_LAYOUT;
  if (M < 1 || N < 8 || N % 8 != 0 || K < 128 || K % 128 != 0) return PURO_ERR_SHAPE;
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31) - 256) return PURO_ERR_SHAPE;
  if (!tiles_fit(M, 128, N, 256)) return PURO_ERR_SHAPE;
  if (!aligned(Aq, 16) || !aligned(Bq, 16) || !aligned(C, 16)) return PURO_ERR_ALIGN;
  if (layout == PURO_WGRAD && !aligned(Bs, 8)) return PURO_ERR_ALIGN;
  if (int d = check_device()) return d;
  return puro::launch_gemm_mx(Aq, As, Bq, Bs, C, M, N, K, layout, stream);
}

int puro_nvfp4_quantize_1x16(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq, int64_t ldq,
                             uint8_t *F, float *amax, puro_stream_t stream) {
  if (X == nullptr || Xq == nullptr || F == nullptr || amax == nullptr) return PURO_ERR_NULL;
  if (R < 1 || C < 16 || C % 16 != 0 || ldx < C || ldq < C / 2) return PURO_ERR_SHAPE;
  if (R > (1ll << 31) - 1 || C > (1ll << 31) - 1) return PURO_ERR_SHAPE;
  if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(F, 16) || !aligned(amax, 4) || ldx % 8 != 0 ||
      ldq % 8 != 0)
    return PURO_ERR_ALIGN;
  if (int d = check_device()) return d;
  return puro::launch_nvfp4_quant_rows(X, R, C, ldx, Xq, ldq, F, amax, stream);
}

int puro_nvfp4_quantize_1x16_transposed(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *XqT,
                                        int64_t ldq, uint8_t *FT, float *amax, puro_stream_t stream) {
  if (X == nullptr || XqT == nullptr || FT == nullptr || amax == nullptr) return PURO_ERR_NULL;
  if (R < 64 || R % 64 != 0 || C < 8 || C % 8 != 0 || ldx < C || ldq < R / 2) return PURO_ERR_SHAPE;
  if (R > (1ll << 31) - 1 || C > (1ll << 31) - 1) return PURO_ERR_SHAPE;
  if (!aligned(X, 16) || !aligned(XqT, 16) || !aligned(FT, 16) || !aligned(amax, 4) || ldx % 8 != 0 ||
      ldq % 16 != 0)
    return PURO_ERR_ALIGN;
  if (int d = check_device()) return d;
  return puro::launch_nvfp4_quant_cols(X, R, C, ldx, XqT, ldq, FT, amax, stream);
}

int puro_nvfp4_quantize_1x16_dual(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                                  int64_t ldq, uint8_t *F, uint8_t *XqT, int64_t ldqt, uint8_t *FT, float *amax,
                                  puro_stream_t stream) {
  if (X == nullptr || Xq == nullptr || F == nullptr || XqT == nullptr || FT == nullptr || amax == nullptr)
    return PURO_ERR_NULL;
  if (R < 64 || R % 64 != 0 || C < 16 || C % 16 != 0 || ldx < C || ldq < C / 2 || ldqt < R / 2)
    return PURO_ERR_SHAPE;
  if (R > (1ll << 31) - 1 || C > (1ll << 31) - 1 || (R / 64) * ((C + 255) / 256) > (1ll << 31) - 1)
    return PURO_ERR_SHAPE;
  if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(F, 16) || !aligned(XqT, 16) || !aligned(FT, 16) ||
      !aligned(amax, 4) || ldx % 8 != 0 || ldq % 8 != 0 || ldqt % 16 != 0)
    return PURO_ERR_ALIGN;
  if (int d = check_device()) return d;
  return puro::launch_nvfp4_quant_dual(X, R, C, ldx, Xq, ldq, F, XqT, ldqt, FT, amax, stream);
}

int puro_nvfp4_gemm(const uint8_t *Aq, const uint8_t *As, const float *a_amax, const uint8_t *Bq,
                    const uint8_t *Bs, const float *b_amax, uint16_t *C, int64_t M, int64_t N, int64_t K,
                    puro_stream_t stream) {
  if (Aq == nullptr || As == nullptr || a_amax == nullptr || Bq == nullptr || Bs == nullptr ||
      b_amax == nullptr || C == nullptr)
    return PURO_ERR_NULL;
  if (M < 1 || N < 8 || N % 8 != 0 || K < 128 || K % 128 != 0) return PURO_ERR_SHAPE;
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31) - 256) return PURO_ERR_SHAPE;
  if (!tiles_fit(M, 128, N, 256)) return PURO_ERR_SHAPE;
  if (!aligned(Aq, 16) || !aligned(Bq, 16) || !aligned(As, 16) || !aligned(Bs, 16) || !aligned(C, 16) ||
      !aligned(a_amax, 4) || !aligned(b_amax, 4))
    return PURO_ERR_ALIGN;
  if (int d = check_device()) return d;
  return puro::launch_gemm_nvfp4(Aq, As, a_amax, Bq, Bs, b_amax, C, M, N, K, stream);
}

int puro_fp8_gemm_blockwise_grouped(const puro_gemm_problem *problems, int count, int layout,
                                    puro_stream_t stream) {
  if (problems == nullptr) return PURO_ERR_NULL;
  if (count < 1 || count > PURO_GROUP_MAX) return PURO_ERR_SHAPE;
  int64_t tiles = 0;
  for (int p = 0; p < count; ++p) {
    const puro_gemm_problem &g = problems[p];
    if (int e = check_gemm(g.Aq, g.As, g.Bq, g.Bs, g.C, g.M, g.N, g.K, layout)) return e;
    tiles += ((g.M + 127) / 128) * ((g.N + 255) / 256);
  }
  if (tiles > (1ll << 31) - (1ll << 16)) return PURO_ERR_SHAPE;
  if (int d = check_device()) return d;
  return puro::launch_gemm_blockwise_grouped(problems, count, layout, stream);
}

int puro_fp8_gemm_blockwise_quant(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                                  const float *Bs, uint16_t *C, uint8_t *Cq, float *Cs, int64_t M,
                                  int64_t N, int64_t K, int layout, puro_stream_t stream) {
  if (Aq == nullptr || As == nullptr || Bq == nullptr || Bs == nullptr || C == nullptr ||
      Cq == nullptr || Cs == nullptr)
    return PURO_ERR_NULL;
  if (layout != PURO_FPROP && layout != PURO_DGRAD) return PURO_ERR_LAYOUT;
  if (M < 1 || N < 128 || N % 128 != 0 || K < 128 || K % 128 != 0) return PURO_ERR_SHAPE;
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31) - 256) return PURO_ERR_SHAPE;
  if (!tiles_fit(M, 128, N, 256)) return PURO_ERR_SHAPE;
  if (!aligned(Aq, 16) || !aligned(Bq, 16) || !aligned(C, 16) || !aligned(Cq, 16) || !aligned(As, 4) ||
      !aligned(Bs, 4) || !aligned(Cs, 4))
    return PURO_ERR_ALIGN;
  if (int d = check_device()) return d;
  return puro::launch_gemm_blockwise_quant(Aq, As, Bq, Bs, C, Cq, Cs, M, N, K, layout, stream);
}

int puro_fp8_gemm_wgrad_acc_f32(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                                const float *Bs, float *C, int64_t M, int64_t N, int64_t K,
                                puro_stream_t stream) {
  if (Aq == nullptr || As == nullptr || Bq == nullptr || Bs == nullptr || C == nullptr)
    return PURO_ERR_NULL;
  if (M < 1 || N < 8 || N % 8 != 0 || K < 128 || K % 128 != 0) return PURO_ERR_SHAPE;
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31) - 256) return PURO_ERR_SHAPE;
  if (!tiles_fit(M, 128, N, 256)) return PURO_ERR_SHAPE;
  if (!aligned(Aq, 16) || !aligned(Bq, 16) || !aligned(C, 16) || !aligned(As, 4) || !aligned(Bs, 4))
    return PURO_ERR_ALIGN;
  if (int d = check_device()) return d;
  return puro::launch_gemm_wgrad_acc_f32(Aq, As, Bq, Bs, C, M, N, K, stream);
}

int puro_fp8_sync_status(puro_stream_t stream) {
  // The status words are per device and collect timeouts from kernels on every stream:
  // join the whole device first so that none is missed.
  if (cudaDeviceSynchronize() != cudaSuccess) return PURO_ERR_CUDA;
  int gemm = 0, quant = 0, mx = 0, nv = 0;
  if (int e = puro::read_and_clear_device_status(stream, &gemm)) return e;
  if (int e = puro::read_and_clear_quant_status(stream, &quant)) return e;
  if (int e = puro::read_and_clear_mx_status(stream, &mx)) return e;
  if (int e = puro::read_and_clear_nv_status(stream, &nv)) return e;
  return (gemm | quant | mx | nv) != 0 ? PURO_ERR_TIMEOUT : PURO_OK;
}

const char *puro_strerror(int status) {
  switch (status) {
    case PURO_OK: return "ok";
    case PURO_ERR_NULL: return "a required pointer is NULL";
    case PURO_ERR_SHAPE: return "invalid size (non-positive, not a multiple of 128 where required, or too large)";
    case PURO_ERR_ALIGN: return "pointer or leading dimension not aligned as required";
    case PURO_ERR_LAYOUT: return "unknown GEMM layout";
    case PURO_ERR_LAUNCH: return "kernel launch failed";
    case PURO_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case PURO_ERR_WORKSPACE: return "workspace too small";
    case PURO_ERR_CUDA: return "CUDA runtime or driver call failed (is there a GPU?)";
    case PURO_ERR_DEVICE: return "the current device is not sm_100 (B200-class)";
    default: return "unknown status";
  }
}

}  // extern "C"
