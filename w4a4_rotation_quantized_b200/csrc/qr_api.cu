// qr_api.cu -- the extern "C" entry points: argument validation on the host,
// then one launch on the caller's stream.  Nothing here allocates memory.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

static_assert(QR_DEV_TIMEOUT_PRODUCER == kDevTimeoutProducer &&
                  QR_DEV_TIMEOUT_WIDEN == kDevTimeoutWiden && QR_DEV_TIMEOUT_MMA == kDevTimeoutMma &&
                  QR_DEV_TIMEOUT_EPILOGUE == kDevTimeoutEpilogue &&
                  QR_DEV_TIMEOUT_DRAIN == kDevTimeoutDrain &&
                  QR_DEV_TIMEOUT_SELFCHECK == kDevTimeoutSelfCheck,
              "status codes of the header and of the kernels");

namespace {

__device__ int32_t g_status_word;   // see qr_device_status()

// Scratch of qr_w4a4_linear_fused_noalloc, one copy per device (a __device__
// array of this library's module, zero when the module loads): the two
// grid-barrier words, then the token rows' scales, zero points, codes and
// outlier copy at their largest sizes.  The barrier count is back at zero
// after every completed call; calls on one device share all of it.
constexpr int64_t kScratchMaxM = 64, kScratchMaxKp = 32768, kScratchMaxOut = 8192;
constexpr size_t kScratchOffScales = 256, kScratchOffZeros = 512, kScratchOffCodes = 1024;
constexpr size_t kScratchOffOut = kScratchOffCodes + kScratchMaxM * kScratchMaxKp / 2;
constexpr size_t kScratchBytes = kScratchOffOut + kScratchMaxM * kScratchMaxOut * 2;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_status_ptr[kMaxDevices] = {};
uint8_t* g_scratch_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
int g_smem[kMaxDevices] = {};

int current_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int32_t* device_status_word() {
  const int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_status_ptr[d] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[d] = static_cast<int32_t*>(p);
  }
  return g_status_ptr[d];
}

// Device address of this device's copy of the no-alloc scratch, or null.
uint8_t* noalloc_scratch() {
  const int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[d] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[d] = static_cast<uint8_t*>(p);
  }
  return g_scratch_ptr[d];
}

int sm_count() {
  const int d = current_device();
  if (d < 0) return 1;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sms[d] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d);
    g_sms[d] = v > 0 ? v : 1;
  }
  return g_sms[d];
}

int max_smem_optin() {
  const int d = current_device();
  if (d < 0) return 48 * 1024;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_smem[d] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, d);
    g_smem[d] = v > 0 ? v : 48 * 1024;
  }
  return g_smem[d];
}

// K_p for a descriptor, or -1.  Shared by qr_packed_k and the row calls.
static int64_t packed_k(const qr_rotation* rot, int64_t K, int32_t n_out) {
  if (rot == nullptr || K < 0 || n_out < 0 || n_out > K) return -1;
  if (!(rot->clip_ratio > 0.0f && rot->clip_ratio <= 1.0f)) return -1;
  const int64_t kr = K - n_out;
  switch (rot->kind) {
    case QR_ROT_NONE:
      return (kr + 127) / 128 * 128;
    case QR_ROT_HADAMARD:
    case QR_ROT_GSR: {
      const int64_t b = rot->block;
      if (!is_pow2(b) || b > 16384) return -1;
      if (rot->kind == QR_ROT_GSR && (b < 2 || b > 256)) return -1;
      const int64_t unit = b > 128 ? b : 128;
      return (kr + unit - 1) / unit * unit;
    }
    case QR_ROT_KRON: {
      const int64_t n1 = rot->n1, n2 = rot->n2;
      if (n1 < 4 || n2 < 4 || n1 % 4 || n2 % 4 || n1 + n2 > 192) return -1;
      if ((n1 * n2) % 128 || kr != n1 * n2) return -1;
      if (rot->p1 == nullptr || rot->p2 == nullptr) return -1;
      if (rot->chan_scale != nullptr && rot->chan_mode != QR_CHAN_DIVIDE &&
          rot->chan_mode != QR_CHAN_MULTIPLY)
        return -1;
      return kr;
    }
    default:
      return -1;
  }
}

static qr_status rows_call(const qr_rotation* rot, const uint16_t* src, int64_t rows, int64_t K,
                           int64_t ld, const int32_t* outlier_idx, int32_t n_out, uint8_t* codes,
                           float* scales, int32_t* zeros, uint16_t* out16, float* rot_debug,
                           qr_stream stream, int bits = 4) {
  if (rot == nullptr || rows < 0 || K < 0 || n_out < 0 || n_out > K) return QR_ERR_INVALID_ARG;
  const int64_t kp = packed_k(rot, K, n_out);
  if (kp < 0) {
    // distinguish malformed from merely unsupported where it is cheap to
    if (rot->kind < QR_ROT_NONE || rot->kind > QR_ROT_KRON) return QR_ERR_INVALID_ARG;
    return (rot->clip_ratio > 0.0f && rot->clip_ratio <= 1.0f) ? QR_ERR_UNSUPPORTED
                                                               : QR_ERR_INVALID_ARG;
  }
  if (rows == 0) return QR_OK;
  if (ld < K || src == nullptr || scales == nullptr) return QR_ERR_INVALID_ARG;
  if (kp > 0 && codes == nullptr) return QR_ERR_INVALID_ARG;
  if (n_out > 0 && (outlier_idx == nullptr || out16 == nullptr)) return QR_ERR_INVALID_ARG;
  if (kp > 32768 || K > 0x7FFFFFFF) return QR_ERR_UNSUPPORTED;
  if (n_out > 0 && (K > 32768 || n_out > 8192)) return QR_ERR_UNSUPPORTED;
  if (kp > 0 && !aligned16(codes)) return QR_ERR_ALIGNMENT;
  if (rot->signs != nullptr) {
    if (rot->kind != QR_ROT_HADAMARD && rot->kind != QR_ROT_GSR) return QR_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(rot->signs) % 8 != 0) return QR_ERR_ALIGNMENT;
  }
  if (zeros != nullptr && rot->kind == QR_ROT_KRON) return QR_ERR_UNSUPPORTED;
  if ((bits == 8 || bits == kFp4Codes) && rot->kind == QR_ROT_KRON) return QR_ERR_UNSUPPORTED;
  if (bits == kFp4Codes && kp > 0 && reinterpret_cast<uintptr_t>(codes) % 32 != 0)
    return QR_ERR_ALIGNMENT;
  RowJob job{};
  job.bits = bits;
  job.src = src;
  job.rows = rows;
  job.K = K;
  job.ld = ld;
  job.outlier_idx = n_out > 0 ? outlier_idx : nullptr;
  job.n_out = n_out;
  job.Kp = static_cast<int32_t>(kp);
  job.Kr = static_cast<int32_t>(K - n_out);
  job.rot = rot;
  job.codes = codes;
  job.scales = scales;
  job.zeros = zeros;
  job.out16 = n_out > 0 ? out16 : nullptr;
  job.rot_debug = rot_debug;
  return launch_rotate_quant(job, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace qr

using namespace qr;

extern "C" {

int32_t qr_abi_version(void) { return QR_ABI_VERSION; }

const char* qr_status_string(qr_status s) {
  switch (s) {
    case QR_OK: return "ok";
    case QR_ERR_INVALID_ARG: return "invalid argument";
    case QR_ERR_UNSUPPORTED: return "unsupported size or kind";
    case QR_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case QR_ERR_CUDA: return "CUDA runtime error";
    case QR_ERR_DEVICE: return "a kernel reported an error";
  }
  return "unknown status";
}

int64_t qr_packed_k(const qr_rotation* rot, int64_t K, int32_t n_out) {
  return packed_k(rot, K, n_out);
}

qr_status qr_rotate_quant(const qr_rotation* rot, const uint16_t* X, int64_t M, int64_t K,
                          int64_t ldx, const int32_t* outlier_idx, int32_t n_out, uint8_t* codes,
                          float* scales, uint16_t* x_out, float* x_rot_debug, qr_stream stream) {
  return rows_call(rot, X, M, K, ldx, outlier_idx, n_out, codes, scales, nullptr, x_out,
                   x_rot_debug, stream);
}

qr_status qr_rotate_quant_asym(const qr_rotation* rot, const uint16_t* X, int64_t M, int64_t K,
                               int64_t ldx, const int32_t* outlier_idx, int32_t n_out,
                               uint8_t* codes, float* scales, int32_t* zeros, uint16_t* x_out,
                               float* x_rot_debug, qr_stream stream) {
  if (zeros == nullptr && M > 0) return QR_ERR_INVALID_ARG;
  return rows_call(rot, X, M, K, ldx, outlier_idx, n_out, codes, scales, zeros, x_out,
                   x_rot_debug, stream);
}

qr_status qr_pack_weights(const qr_rotation* rot_w, const uint16_t* W, int64_t N, int64_t K,
                          int64_t ldw, const int32_t* outlier_idx, int32_t n_out, uint8_t* w_codes,
                          float* w_scales, uint16_t* w_out, float* w_rot_debug, qr_stream stream) {
  return rows_call(rot_w, W, N, K, ldw, outlier_idx, n_out, w_codes, w_scales, nullptr, w_out,
                   w_rot_debug, stream);
}

qr_status qr_weight_code_sums(const uint8_t* w_codes, int64_t N, int64_t K_p, int32_t* w_sums,
                              qr_stream stream) {
  if (N < 0 || K_p < 0 || K_p % 128 != 0) return QR_ERR_INVALID_ARG;
  if (N == 0) return QR_OK;
  if (w_sums == nullptr || (K_p > 0 && w_codes == nullptr)) return QR_ERR_INVALID_ARG;
  if (K_p > 0 && !aligned16(w_codes)) return QR_ERR_ALIGNMENT;
  return launch_code_row_sums(w_codes, N, K_p, w_sums, reinterpret_cast<cudaStream_t>(stream));
}

qr_status qr_kv_quantize(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t tokens,
                         int32_t heads, int32_t head_dim, int32_t group, uint16_t* q_rot,
                         uint8_t* k_codes, float* k_scales, int32_t* k_zeros, uint8_t* v_codes,
                         float* v_scales, int32_t* v_zeros, qr_stream stream) {
  if (tokens < 0 || heads <= 0 || group <= 0) return QR_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128 && head_dim != 256)
    return QR_ERR_UNSUPPORTED;
  const int64_t width = static_cast<int64_t>(heads) * head_dim;
  if ((group != 128 && group != 256) || group % head_dim != 0 || width % group != 0)
    return QR_ERR_UNSUPPORTED;
  // each side is all there or all absent
  if ((Q == nullptr) != (q_rot == nullptr)) return QR_ERR_INVALID_ARG;
  const bool k_any = K || k_codes || k_scales || k_zeros, k_all = K && k_codes && k_scales && k_zeros;
  const bool v_any = V || v_codes || v_scales || v_zeros, v_all = V && v_codes && v_scales && v_zeros;
  if (k_any != k_all || v_any != v_all) return QR_ERR_INVALID_ARG;
  if (tokens == 0) return QR_OK;
  if (Q != nullptr && (!aligned16(Q) || !aligned16(q_rot))) return QR_ERR_ALIGNMENT;
  if (tokens * width > (int64_t(1) << 40)) return QR_ERR_UNSUPPORTED;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // keys and values: rows of `group` values, one quantization group each,
  // one warp per group
  const int64_t rows = tokens * (width / group);
  if ((k_all && (!aligned16(K) || !aligned16(k_codes))) ||
      (v_all && (!aligned16(V) || !aligned16(v_codes))))
    return QR_ERR_ALIGNMENT;
  qr_status st = QR_OK;
  if (k_all) st = launch_kv_group_quant(K, rows, group, head_dim, true, k_codes, k_scales, k_zeros, s);
  if (st == QR_OK && v_all)
    st = launch_kv_group_quant(V, rows, group, head_dim, false, v_codes, v_scales, v_zeros, s);
  if (st == QR_OK && Q != nullptr) st = launch_head_rotate(Q, q_rot, tokens * heads, head_dim, s);
  return st;
}

}  // extern "C"

namespace qr {

static qr_status linear_call(const uint8_t* a_codes, const float* a_scales, const int32_t* a_zeros,
                             const uint8_t* w_codes, const float* w_scales, const int32_t* w_sums,
                             int64_t M, int64_t N, int64_t K_p, const uint16_t* x_out,
                             const uint16_t* w_out, int32_t n_out, uint16_t* Y, int64_t ldy,
                             int32_t* acc_debug, qr_stream stream, int bits = 4) {
  if (M < 0 || N < 0 || K_p < 0 || n_out < 0) return QR_ERR_INVALID_ARG;
  if (K_p % 128 != 0) return QR_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return QR_OK;
  if (Y == nullptr || ldy < N || a_scales == nullptr || w_scales == nullptr)
    return QR_ERR_INVALID_ARG;
  if (K_p > 0 && (a_codes == nullptr || w_codes == nullptr)) return QR_ERR_INVALID_ARG;
  if (n_out > 0 && (x_out == nullptr || w_out == nullptr)) return QR_ERR_INVALID_ARG;
  if (K_p > 65536 || M > 0x7FFFFFFF || N > 0x7FFFFFFF) return QR_ERR_UNSUPPORTED;
  if (n_out % 8 != 0) return QR_ERR_UNSUPPORTED;
  if (K_p > 0 && (!aligned16(a_codes) || !aligned16(w_codes))) return QR_ERR_ALIGNMENT;
  if (bits == kFp4Codes && K_p > 0 &&     // the 4-bit tensor maps want 32-byte bases
      (reinterpret_cast<uintptr_t>(a_codes) % 32 != 0 || reinterpret_cast<uintptr_t>(w_codes) % 32 != 0))
    return QR_ERR_ALIGNMENT;
  if (n_out > 0 && (!aligned16(x_out) || !aligned16(w_out))) return QR_ERR_ALIGNMENT;
  GemmJob j{};
  j.a_codes = a_codes;
  j.a_scales = a_scales;
  j.a_zeros = a_zeros;
  j.w_codes = w_codes;
  j.w_scales = w_scales;
  j.w_sums = w_sums;
  j.M = M;
  j.N = N;
  j.Kp = K_p;
  j.x_out = n_out > 0 ? x_out : nullptr;
  j.w_out = n_out > 0 ? w_out : nullptr;
  j.n_out = n_out;
  j.Y = Y;
  j.ldy = ldy;
  j.acc_debug = acc_debug;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return bits == 8 ? launch_w8a8_gemm(j, st) : bits == kFp4Codes ? launch_fp4_gemm(j, st)
                                                                 : launch_w4a4_gemm(j, st);
}

}  // namespace qr

extern "C" {

qr_status qr_w4a4_linear(const uint8_t* a_codes, const float* a_scales, const uint8_t* w_codes,
                         const float* w_scales, int64_t M, int64_t N, int64_t K_p,
                         const uint16_t* x_out, const uint16_t* w_out, int32_t n_out, uint16_t* Y,
                         int64_t ldy, int32_t* acc_debug, qr_stream stream) {
  return linear_call(a_codes, a_scales, nullptr, w_codes, w_scales, nullptr, M, N, K_p, x_out,
                     w_out, n_out, Y, ldy, acc_debug, stream);
}

qr_status qr_w4a4_linear_asym(const uint8_t* a_codes, const float* a_scales,
                              const int32_t* a_zeros, const uint8_t* w_codes,
                              const float* w_scales, const int32_t* w_sums, int64_t M, int64_t N,
                              int64_t K_p, const uint16_t* x_out, const uint16_t* w_out,
                              int32_t n_out, uint16_t* Y, int64_t ldy, int32_t* acc_debug,
                              qr_stream stream) {
  if (M > 0 && N > 0 && (a_zeros == nullptr || w_sums == nullptr)) return QR_ERR_INVALID_ARG;
  return linear_call(a_codes, a_scales, a_zeros, w_codes, w_scales, w_sums, M, N, K_p, x_out,
                     w_out, n_out, Y, ldy, acc_debug, stream);
}

}  // extern "C"

namespace qr {

// Shared by qr_w4a4_linear_fused and its no-alloc form: with `noalloc`, the
// token rows' codes, scales, zero points and outlier copy and the barrier
// words live in this device's scratch (resolved after the arguments pass;
// a_zeros is then only a flag: non-null for asymmetric activations).
static qr_status fused_call(const qr_rotation* rot, const uint16_t* X, int64_t M, int64_t K,
                            int64_t ldx, const int32_t* outlier_idx, int32_t n_out,
                            const uint8_t* w_codes, const float* w_scales, const int32_t* w_sums,
                            const uint16_t* w_out, int64_t N, uint8_t* a_codes, float* a_scales,
                            int32_t* a_zeros, uint16_t* x_out, uint16_t* Y, int64_t ldy,
                            uint32_t* sync, qr_stream stream, bool noalloc) {
  if (rot == nullptr || M < 0 || N < 0 || K < 0 || n_out < 0 || n_out > K) return QR_ERR_INVALID_ARG;
  const int64_t kp = packed_k(rot, K, n_out);
  if (kp < 0) {
    if (rot->kind < QR_ROT_NONE || rot->kind > QR_ROT_KRON) return QR_ERR_INVALID_ARG;
    return (rot->clip_ratio > 0.0f && rot->clip_ratio <= 1.0f) ? QR_ERR_UNSUPPORTED
                                                               : QR_ERR_INVALID_ARG;
  }
  if (M == 0 || N == 0) return QR_OK;
  if (X == nullptr || ldx < K || (!noalloc && a_scales == nullptr) || w_scales == nullptr ||
      Y == nullptr || ldy < N || (!noalloc && sync == nullptr))
    return QR_ERR_INVALID_ARG;
  if (kp > 0 && ((!noalloc && a_codes == nullptr) || w_codes == nullptr)) return QR_ERR_INVALID_ARG;
  if (n_out > 0 && (outlier_idx == nullptr || (!noalloc && x_out == nullptr) || w_out == nullptr))
    return QR_ERR_INVALID_ARG;
  if (a_zeros != nullptr && w_sums == nullptr) return QR_ERR_INVALID_ARG;
  if (rot->signs != nullptr) {
    if (rot->kind != QR_ROT_HADAMARD && rot->kind != QR_ROT_GSR) return QR_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(rot->signs) % 8 != 0) return QR_ERR_ALIGNMENT;
  }
  if (M > 64 || rot->kind == QR_ROT_KRON) return QR_ERR_UNSUPPORTED;
  if (kp > 32768 || K > 32768 || n_out > 8192 || N > 0x7FFFFFFF) return QR_ERR_UNSUPPORTED;
  if (n_out % 8 != 0) return QR_ERR_UNSUPPORTED;
  if (noalloc) {
    if (M > kScratchMaxM || kp > kScratchMaxKp || n_out > kScratchMaxOut) return QR_ERR_UNSUPPORTED;
    uint8_t* sc = noalloc_scratch();
    if (sc == nullptr) return QR_ERR_CUDA;
    sync = reinterpret_cast<uint32_t*>(sc);
    a_scales = reinterpret_cast<float*>(sc + kScratchOffScales);
    a_zeros = a_zeros != nullptr ? reinterpret_cast<int32_t*>(sc + kScratchOffZeros) : nullptr;
    a_codes = sc + kScratchOffCodes;
    x_out = reinterpret_cast<uint16_t*>(sc + kScratchOffOut);
  }
  if (kp > 0 && (!aligned16(a_codes) || !aligned16(w_codes))) return QR_ERR_ALIGNMENT;
  if (n_out > 0 && (!aligned16(x_out) || !aligned16(w_out))) return QR_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(sync) % 8 != 0) return QR_ERR_ALIGNMENT;
  RowJob r{};
  r.bits = 4;
  r.src = X;
  r.rows = M;
  r.K = K;
  r.ld = ldx;
  r.outlier_idx = n_out > 0 ? outlier_idx : nullptr;
  r.n_out = n_out;
  r.Kp = static_cast<int32_t>(kp);
  r.Kr = static_cast<int32_t>(K - n_out);
  r.rot = rot;
  r.codes = a_codes;
  r.scales = a_scales;
  r.zeros = a_zeros;
  r.out16 = n_out > 0 ? x_out : nullptr;
  GemmJob j{};
  j.a_codes = a_codes;
  j.a_scales = a_scales;
  j.a_zeros = a_zeros;
  j.w_codes = w_codes;
  j.w_scales = w_scales;
  j.w_sums = a_zeros != nullptr ? w_sums : nullptr;
  j.M = M;
  j.N = N;
  j.Kp = kp;
  j.x_out = n_out > 0 ? x_out : nullptr;
  j.w_out = n_out > 0 ? w_out : nullptr;
  j.n_out = n_out;
  j.Y = Y;
  j.ldy = ldy;
  return launch_w4a4_decode_fused(j, r, sync, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace qr

extern "C" {

qr_status qr_w4a4_linear_fused(const qr_rotation* rot, const uint16_t* X, int64_t M, int64_t K,
                               int64_t ldx, const int32_t* outlier_idx, int32_t n_out,
                               const uint8_t* w_codes, const float* w_scales, const int32_t* w_sums,
                               const uint16_t* w_out, int64_t N, uint8_t* a_codes, float* a_scales,
                               int32_t* a_zeros, uint16_t* x_out, uint16_t* Y, int64_t ldy,
                               uint32_t* sync, qr_stream stream) {
  return fused_call(rot, X, M, K, ldx, outlier_idx, n_out, w_codes, w_scales, w_sums, w_out, N,
                    a_codes, a_scales, a_zeros, x_out, Y, ldy, sync, stream, false);
}

qr_status qr_w4a4_linear_fused_noalloc(const qr_rotation* rot, const uint16_t* X, int64_t M,
                                       int64_t K, int64_t ldx, const int32_t* outlier_idx,
                                       int32_t n_out, const uint8_t* w_codes,
                                       const float* w_scales, const int32_t* w_sums,
                                       const uint16_t* w_out, int64_t N, int32_t asym,
                                       uint16_t* Y, int64_t ldy, qr_stream stream) {
  static int32_t flag = 1;                  // any non-null pointer selects zero points
  return fused_call(rot, X, M, K, ldx, outlier_idx, n_out, w_codes, w_scales, w_sums, w_out, N,
                    nullptr, nullptr, asym ? &flag : nullptr, nullptr, Y, ldy, nullptr, stream,
                    true);
}

qr_status qr_select_outliers(const uint16_t* X_calib, int64_t T, int64_t K, int64_t ldx,
                             int32_t k, int32_t* idx_out, qr_stream stream) {
  if (T < 0 || K < 1 || k < 0 || k > K || ldx < K) return QR_ERR_INVALID_ARG;
  if (k > 0 && (idx_out == nullptr || (T > 0 && X_calib == nullptr))) return QR_ERR_INVALID_ARG;
  if (K > 16384) return QR_ERR_UNSUPPORTED;
  return launch_select_outliers(X_calib, T, K, ldx, k, idx_out,
                                reinterpret_cast<cudaStream_t>(stream));
}

qr_status qr_invert_transpose(const float* P, int32_t n, float* out, int32_t* info,
                              qr_stream stream) {
  if (P == nullptr || out == nullptr || info == nullptr || n < 1) return QR_ERR_INVALID_ARG;
  if (n > 128) return QR_ERR_UNSUPPORTED;
  return launch_invert_transpose(P, n, out, info, reinterpret_cast<cudaStream_t>(stream));
}

qr_status qr_rotate_quant8(const qr_rotation* rot, const uint16_t* X, int64_t M, int64_t K,
                           int64_t ldx, const int32_t* outlier_idx, int32_t n_out, int8_t* codes,
                           float* scales, uint16_t* x_out, float* x_rot_debug, qr_stream stream) {
  return rows_call(rot, X, M, K, ldx, outlier_idx, n_out, reinterpret_cast<uint8_t*>(codes), scales,
                   nullptr, x_out, x_rot_debug, stream, 8);
}

qr_status qr_pack_weights8(const qr_rotation* rot_w, const uint16_t* W, int64_t N, int64_t K,
                           int64_t ldw, const int32_t* outlier_idx, int32_t n_out, int8_t* w_codes,
                           float* w_scales, uint16_t* w_out, float* w_rot_debug, qr_stream stream) {
  return rows_call(rot_w, W, N, K, ldw, outlier_idx, n_out, reinterpret_cast<uint8_t*>(w_codes),
                   w_scales, nullptr, w_out, w_rot_debug, stream, 8);
}

qr_status qr_w8a8_linear(const int8_t* a_codes, const float* a_scales, const int8_t* w_codes,
                         const float* w_scales, int64_t M, int64_t N, int64_t K_p,
                         const uint16_t* x_out, const uint16_t* w_out, int32_t n_out, uint16_t* Y,
                         int64_t ldy, int32_t* acc_debug, qr_stream stream) {
  return linear_call(reinterpret_cast<const uint8_t*>(a_codes), a_scales, nullptr,
                     reinterpret_cast<const uint8_t*>(w_codes), w_scales, nullptr, M, N, K_p,
                     x_out, w_out, n_out, Y, ldy, acc_debug, stream, 8);
}

qr_status qr_rotate_quant_fp4(const qr_rotation* rot, const uint16_t* X, int64_t M, int64_t K,
                              int64_t ldx, const int32_t* outlier_idx, int32_t n_out,
                              uint8_t* codes, float* scales, uint16_t* x_out, float* x_rot_debug,
                              qr_stream stream) {
  return rows_call(rot, X, M, K, ldx, outlier_idx, n_out, codes, scales, nullptr, x_out,
                   x_rot_debug, stream, kFp4Codes);
}

qr_status qr_pack_weights_fp4(const qr_rotation* rot_w, const uint16_t* W, int64_t N, int64_t K,
                              int64_t ldw, const int32_t* outlier_idx, int32_t n_out,
                              uint8_t* w_codes, float* w_scales, uint16_t* w_out,
                              float* w_rot_debug, qr_stream stream) {
  return rows_call(rot_w, W, N, K, ldw, outlier_idx, n_out, w_codes, w_scales, nullptr, w_out,
                   w_rot_debug, stream, kFp4Codes);
}

qr_status qr_fp4_linear(const uint8_t* a_codes, const float* a_scales, const uint8_t* w_codes,
                        const float* w_scales, int64_t M, int64_t N, int64_t K_p,
                        const uint16_t* x_out, const uint16_t* w_out, int32_t n_out, uint16_t* Y,
                        int64_t ldy, float* acc_debug, qr_stream stream) {
  return linear_call(a_codes, a_scales, nullptr, w_codes, w_scales, nullptr, M, N, K_p, x_out,
                     w_out, n_out, Y, ldy, reinterpret_cast<int32_t*>(acc_debug), stream,
                     kFp4Codes);
}

qr_status qr_check_wait_timeout(int64_t limit_ns, qr_stream stream) {
  if (limit_ns < 1000 || limit_ns > 100000000) return QR_ERR_INVALID_ARG;
  return launch_wait_selfcheck(static_cast<uint64_t>(limit_ns),
                               reinterpret_cast<cudaStream_t>(stream));
}

qr_status qr_device_status(int32_t* code_out) {
  if (code_out == nullptr) return QR_ERR_INVALID_ARG;
  *code_out = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return QR_ERR_CUDA;
  int32_t* p = device_status_word();
  if (p == nullptr) return QR_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return QR_ERR_CUDA;
  if (v != 0) {
    const int32_t zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return QR_ERR_CUDA;
  }
  *code_out = v;
  return QR_OK;
}

}  // extern "C"
