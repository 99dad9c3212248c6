// kv_cache.cu -- the query side of the KV-cache rotation R3.
//
// SpinQuant (review answer of reviewer brBn, Q2/A2) applies the same R3 to
// the query and key rows of every head after RoPE, so that
// (q R3)(k R3)^T = q k^T; here R3 is the normalized Hadamard of the head
// dimension.  The keys are rotated and quantized group-wise (groups of 128,
// asymmetric 4-bit, the KV-cache setting of FlatQuant §3) by
// kv_group_quant_kernel in rotate_quant.cu, one warp per group; the queries
// stay fp16 and only need the rotation, which this kernel does.
//
// One warp per head vector of D = 32 E elements: lane L holds elements
// [E L, E L + E) (one vector load), the low log2(E) butterfly stages run in
// registers, the five stages over the lane bits by xor shuffles; the
// 1/sqrt(D) factor is applied before the fp16 conversion.
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

template <int E>
struct HalfVec;
template <> struct HalfVec<1> { using T = __half; };
template <> struct HalfVec<2> { using T = uint32_t; };
template <> struct HalfVec<4> { using T = uint2; };
template <> struct HalfVec<8> { using T = uint4; };

constexpr int kBatch = 4;

template <int E>
__global__ void __launch_bounds__(256) head_rotate_kernel(const __half* __restrict__ src,
                                                          __half* __restrict__ dst,
                                                          int64_t vectors, float scale) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int D = 32 * E;
  constexpr int LE = E == 1 ? 0 : E == 2 ? 1 : E == 4 ? 2 : 3;
  using V = typename HalfVec<E>::T;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // kBatch head vectors per warp and iteration, their loads issued together
  for (int64_t v0 = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * kBatch;
       v0 < vectors; v0 += nwarps * kBatch) {
    V raws[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (v0 + u < vectors) raws[u] = *reinterpret_cast<const V*>(src + (v0 + u) * D + lane * E);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t v = v0 + u;
      if (v >= vectors) break;                       // uniform over the warp
      const V raw = raws[u];
      const __half* h = reinterpret_cast<const __half*>(&raw);
      float x[E];
#pragma unroll
      for (int j = 0; j < E; ++j) x[j] = __half2float(h[j]);
      // stages on the element bits held by the thread
#pragma unroll
      for (int b = 0; b < LE; ++b)
#pragma unroll
        for (int j = 0; j < E; ++j)
          if (!(j & (1 << b))) {
            const float a = x[j], c = x[j | (1 << b)];
            x[j] = a + c;
            x[j | (1 << b)] = a - c;
          }
      // stages on the lane bits: the partner lane holds the other element
#pragma unroll
      for (int lb = 0; lb < 5; ++lb) {
        const bool upper = (lane >> lb) & 1;
#pragma unroll
        for (int j = 0; j < E; ++j) {
          const float o = __shfl_xor_sync(0xffffffffu, x[j], 1 << lb);
          x[j] = upper ? o - x[j] : x[j] + o;
        }
      }
      V out;
      __half* oh = reinterpret_cast<__half*>(&out);
#pragma unroll
      for (int j = 0; j < E; ++j) oh[j] = __float2half_rn(x[j] * scale);
      *reinterpret_cast<V*>(dst + v * D + lane * E) = out;
    }
  }
}

template <int E>
cudaError_t run_head_rotate(const uint16_t* src, uint16_t* dst, int64_t vectors,
                            cudaStream_t stream) {
  constexpr int kWarps = 8;
  const int64_t blocks = std::min<int64_t>((vectors + kWarps * kBatch - 1) / (kWarps * kBatch),
                                           static_cast<int64_t>(sm_count()) * 8);
  const float scale = static_cast<float>(1.0 / std::sqrt(32.0 * E));
  return launch_pdl(head_rotate_kernel<E>, dim3(static_cast<unsigned>(blocks)), dim3(32 * kWarps),
                    0, stream, 1, reinterpret_cast<const __half*>(src),
                    reinterpret_cast<__half*>(dst), vectors, scale);
}

}  // namespace

qr_status launch_head_rotate(const uint16_t* src, uint16_t* dst, int64_t vectors, int head_dim,
                             cudaStream_t stream) {
  if (vectors == 0) return QR_OK;
  cudaError_t e;
  switch (head_dim) {
    case 32: e = run_head_rotate<1>(src, dst, vectors, stream); break;
    case 64: e = run_head_rotate<2>(src, dst, vectors, stream); break;
    case 128: e = run_head_rotate<4>(src, dst, vectors, stream); break;
    case 256: e = run_head_rotate<8>(src, dst, vectors, stream); break;
    default: return QR_ERR_UNSUPPORTED;
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
