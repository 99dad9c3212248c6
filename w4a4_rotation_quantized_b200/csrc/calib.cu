// calib.cu -- offline helpers: QUIK outlier-column selection, the inverse
// transpose of a Kronecker factor (both once per layer, in one CTA), and the
// per-row sums of packed weight codes that the asymmetric-activation
// epilogue needs.
#include <cuda_fp16.h>

#include "qr_internal.h"

namespace qr {

namespace {

constexpr int kSelThreads = 1024;

// QUIK ("QUIK：LLM上的一种4-bit推理方法", §3): the outlier columns are the k
// columns with the largest infinity-norm over the calibration batch.  Keys
// pack (norm bits, ~column) so that one descending bitonic sort orders by
// norm and, among equal norms, by ascending column; the k winners are then
// written out in ascending column order through a flag scan.
__global__ void __launch_bounds__(kSelThreads) select_outliers_kernel(
    const __half* __restrict__ x, int64_t T, int K, int64_t ld, int k, int P,
    int32_t* __restrict__ idx_out) {
  extern __shared__ __align__(16) uint8_t smem[];
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smem);   // [P]
  int* cnt = reinterpret_cast<int*>(smem);                                   // reused after sort
  const int tid = threadIdx.x;

  for (int c = tid; c < P; c += blockDim.x) {
    unsigned long long kv = 0;
    if (c < K) {
      float m = 0.0f;
      for (int64_t t = 0; t < T; ++t) m = fmaxf(m, fabsf(__half2float(x[t * ld + c])));
      kv = (static_cast<unsigned long long>(__float_as_uint(m)) << 32) |
           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<unsigned>(c));
    }
    key[c] = kv;
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = key[i], b = key[j];
          if (desc ? (a < b) : (a > b)) { key[i] = b; key[j] = a; }
        }
      }
      __syncthreads();
    }
  }
  // flag the winners by column
  __shared__ unsigned int flag_words[512];          // K <= 16384 bits
  for (int w = tid; w < 512; w += blockDim.x) flag_words[w] = 0;
  __syncthreads();
  for (int i = tid; i < k; i += blockDim.x) {
    const unsigned c = 0xFFFFFFFFu - static_cast<unsigned>(key[i] & 0xFFFFFFFFull);
    atomicOr(&flag_words[c >> 5], 1u << (c & 31));
  }
  __syncthreads();
  // ascending compaction: thread t owns columns [t*per, (t+1)*per)
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int c0 = tid * per, c1 = min(K, c0 + per);
  int mine = 0;
  for (int c = c0; c < c1; ++c) mine += (flag_words[c >> 5] >> (c & 31)) & 1;
  cnt[tid] = mine;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int t = 0; t < static_cast<int>(blockDim.x); ++t) { const int v = cnt[t]; cnt[t] = run; run += v; }
  }
  __syncthreads();
  int pos = cnt[tid];
  for (int c = c0; c < c1; ++c)
    if ((flag_words[c >> 5] >> (c & 31)) & 1) idx_out[pos++] = c;
}

constexpr int kInvThreads = 256;

// out = (P^{-1})^T by Gauss-Jordan elimination with partial pivoting, in
// place, in fp64 (FlatQuant §2.3: the weights take the inverse transform).
// Row swaps are recorded and undone as column swaps at the end.
__global__ void __launch_bounds__(kInvThreads) invert_transpose_kernel(
    const float* __restrict__ P, int n, float* __restrict__ out, int32_t* __restrict__ info) {
  extern __shared__ __align__(16) uint8_t smem[];
  double* A = reinterpret_cast<double*>(smem);                 // [n x n]
  double* fcol = A + n * n;                                     // [n]
  int* piv = reinterpret_cast<int*>(fcol + n);                  // [n]
  __shared__ int s_pivot;
  __shared__ int s_fail;
  const int tid = threadIdx.x;
  for (int i = tid; i < n * n; i += blockDim.x) A[i] = static_cast<double>(P[i]);
  if (tid == 0) s_fail = 0;
  __syncthreads();

  for (int k = 0; k < n; ++k) {
    if (tid == 0) {
      int best = k;
      double bv = fabs(A[k * n + k]);
      for (int i = k + 1; i < n; ++i) {
        const double v = fabs(A[i * n + k]);
        if (v > bv) { bv = v; best = i; }
      }
      s_pivot = best;
      piv[k] = best;
      if (!(bv > 0.0)) s_fail = k + 1;
    }
    __syncthreads();
    if (s_fail) break;
    const int pr = s_pivot;
    if (pr != k)
      for (int j = tid; j < n; j += blockDim.x) {
        const double t = A[k * n + j]; A[k * n + j] = A[pr * n + j]; A[pr * n + j] = t;
      }
    __syncthreads();
    const double d = A[k * n + k];
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x) A[k * n + j] = (j == k ? 1.0 : A[k * n + j]) / d;
    for (int i = tid; i < n; i += blockDim.x) fcol[i] = (i == k) ? 0.0 : A[i * n + k];
    __syncthreads();
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int i = e / n, j = e - i * n;
      if (i == k) continue;
      const double base = (j == k) ? 0.0 : A[e];
      A[e] = base - fcol[i] * A[k * n + j];
    }
    __syncthreads();
  }
  if (s_fail) {
    if (tid == 0) *info = s_fail;
    return;
  }
  for (int k = n - 1; k >= 0; --k) {
    const int pr = piv[k];
    if (pr != k)
      for (int i = tid; i < n; i += blockDim.x) {
        const double t = A[i * n + k]; A[i * n + k] = A[i * n + pr]; A[i * n + pr] = t;
      }
    __syncthreads();
  }
  for (int e = tid; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e - i * n;
    out[j * n + i] = static_cast<float>(A[e]);     // transpose
  }
  if (tid == 0) *info = 0;
}

// Row sums of packed signed 4-bit codes: sums[row] = sum_k q[row, k].  With
// asymmetric activations s_a (q_a - z_a) the GEMM's integer product of the
// stored codes needs - z_a * sums[n] (QUIK §1: activations asymmetric per
// token).  One warp per row, 16 bytes (32 codes) per lane per step.
__global__ void __launch_bounds__(256) code_row_sums_kernel(const uint8_t* __restrict__ codes,
                                                            int64_t rows, int64_t row_bytes,
                                                            int32_t* __restrict__ sums) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint8_t* r = codes + row * row_bytes;
  int32_t acc = 0;
  for (int64_t b = 16 * lane; b < row_bytes; b += 16 * 32) {
    const uint4 u = *reinterpret_cast<const uint4*>(r + b);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j)                       // sign-extend each nibble
        acc += static_cast<int32_t>(w[i] << (28 - 4 * j)) >> 28;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) sums[row] = acc;
}

}  // namespace

qr_status launch_code_row_sums(const uint8_t* codes, int64_t rows, int64_t kp, int32_t* sums,
                               cudaStream_t stream) {
  if (rows == 0) return QR_OK;
  const int64_t blocks = (rows + 7) / 8;
  code_row_sums_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(codes, rows, kp / 2, sums);
  return cudaGetLastError() == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

qr_status launch_select_outliers(const uint16_t* x, int64_t T, int64_t K, int64_t ld, int32_t k,
                                 int32_t* idx_out, cudaStream_t stream) {
  if (k == 0) return QR_OK;
  int P = 1;
  while (P < K) P <<= 1;
  const size_t smem = sizeof(unsigned long long) * static_cast<size_t>(P);
  if (smem > static_cast<size_t>(max_smem_optin())) return QR_ERR_UNSUPPORTED;
  cudaError_t e = cudaFuncSetAttribute(select_outliers_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return QR_ERR_CUDA;
  select_outliers_kernel<<<1, kSelThreads, smem, stream>>>(
      reinterpret_cast<const __half*>(x), T, static_cast<int>(K), ld, k, P, idx_out);
  return cudaGetLastError() == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

qr_status launch_invert_transpose(const float* P, int32_t n, float* out, int32_t* info,
                                  cudaStream_t stream) {
  const size_t smem = sizeof(double) * (static_cast<size_t>(n) * n + n) + sizeof(int) * n;
  if (smem > static_cast<size_t>(max_smem_optin())) return QR_ERR_UNSUPPORTED;
  cudaError_t e = cudaFuncSetAttribute(invert_transpose_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return QR_ERR_CUDA;
  invert_transpose_kernel<<<1, kInvThreads, smem, stream>>>(P, n, out, info);
  return cudaGetLastError() == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
