// w4a4_gemm.cu -- the W4A4 linear on fifth-generation tensor cores: dispatch
// and the host-side tensor-map helper shared by its kernels.
//
//   acc[m, n] = sum_k qa[m, k] qw[n, k]                    (int32, exact)
//   Y[m, n]   = fp16( acc * sa[m] * sw[n] + X_out[m] . W_out[n] )
//
// QUIK ("QUIK：LLM上的一种4-bit推理方法", §1 workflow, §4 inference): the
// INT4 product of the non-outlier columns runs on integer tensor cores with
// INT32 accumulation, is dequantized to fp16 and added to the fp16 product of
// the outlier columns.  FlatQuant §3 / QuaRot: per-token x per-channel
// symmetric scales, so the dequantization is one multiply per output.
//
// sm_100a has no 4-bit integer MMA, so packed codes are staged by TMA into
// shared memory, widened there to 8-bit by dedicated warps, and multiplied by
// tcgen05.mma kind::i8 into an int32 accumulator in tensor memory.  Widening
// puts each nibble in the HIGH half of a byte: the byte read as int8 is then
// exactly 16*q, so no sign extension is needed and the accumulator holds
// 256*acc (|256*acc| <= 256*49*65536 < 2^31).  The 32 codes of a 16-byte
// packed chunk are written as two 16-byte chunks, even elements then odd
// elements; A and B use the same order, which leaves every dot product
// unchanged.
//
// Two kernels:
//   M > 64   w4a4_gemm_pair.cu: CTA pairs (tcgen05 cta_group::2), 256-row
//            activation tiles widened into tensor memory, weights in shared
//            memory, persistent over tiles.
//   M <= 64  w4a4_gemm_decode.cu: weight rows on the MMA M side (widened into
//            tensor memory), tokens on the N side, K split over a cluster.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "qr_internal.h"

namespace qr {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Row-major 2-D tensor of `rows` rows, `cols` elements per row, row pitch
// `pitch_bytes`; box of box_cols x box_rows elements.
bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr,
                        uint64_t cols, uint64_t rows, uint64_t pitch_bytes, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  // (no L2 promotion for the packed 4-bit element type)
  const bool packed4 = dtype == CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
  return fn(map, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            packed4 ? CU_TENSOR_MAP_L2_PROMOTION_NONE : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

qr_status launch_w4a4_gemm(const GemmJob& j, cudaStream_t stream) {
  if (j.M == 0 || j.N == 0) return QR_OK;
  if (j.M <= 64) return launch_w4a4_gemm_decode(j, stream);
  return launch_w4a4_gemm_pair(j, stream);
}

}  // namespace qr
