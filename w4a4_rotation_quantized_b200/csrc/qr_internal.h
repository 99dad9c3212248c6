// qr_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/qr.h"

#include <utility>

namespace qr {

// Launches kernel `k` with programmatic dependent launch allowed (its CTAs
// may start while the previous kernel on the stream finishes; the kernel
// calls grid_dep_wait before touching global memory) and, when cluster_x >
// 1, a runtime cluster of cluster_x CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// Device address of this device's status word (see qr_device_status).
int32_t* device_status_word();

// Number of SMs of the current device (cached).
int sm_count();

// Maximum opt-in dynamic shared memory per block of the current device.
int max_smem_optin();

// Parameters of the row kernels (rotate + quantize one matrix row by row);
// used for activations (kernel a) and weights (kernel c) alike.
struct RowJob {
  const uint16_t* src;        // fp16 [rows x ld]
  int64_t rows, K, ld;
  const int32_t* outlier_idx; // [n_out] or null
  int32_t n_out;
  int32_t Kp;                 // packed width
  int32_t Kr;                 // K - n_out, the rotated columns
  const qr_rotation* rot;
  uint8_t* codes;             // [rows x Kp/2]
  float* scales;              // [rows]
  int32_t* zeros;             // [rows] zero points (asymmetric activations) or null
  uint16_t* out16;            // [rows x n_out] or null
  float* rot_debug;           // [rows x Kp] or null
  int32_t bits;               // codes: 4 (int4 nibbles), 8 (one int8 each) or kFp4Codes
};

// RowJob::bits for e2m1 codes, packed two per byte like the int4 nibbles.
constexpr int32_t kFp4Codes = 0xF4;

qr_status launch_rotate_quant(const RowJob& job, cudaStream_t stream);

// FlatQuant Kronecker transform on tensor cores (n1 = 128, n2 = 64, no
// outlier split, aligned rows); other Kronecker shapes run on CUDA cores.
bool kron_tc_supported(const RowJob& job);
qr_status launch_kron_tc(const RowJob& job, cudaStream_t stream);

struct GemmJob {
  const uint8_t* a_codes; const float* a_scales;
  const int32_t* a_zeros;     // asymmetric activations: zero points [M], else null
  const uint8_t* w_codes; const float* w_scales;
  const int32_t* w_sums;      // with a_zeros: per weight row, the sum of its codes [N]
  int64_t M, N, Kp;
  const uint16_t* x_out; const uint16_t* w_out; int32_t n_out;
  uint16_t* Y; int64_t ldy;
  int32_t* acc_debug;
};

qr_status launch_w4a4_gemm(const GemmJob& job, cudaStream_t stream);

// 8-bit codes (one int8 per code, rows of K_p bytes): TMA-fed tcgen05
// kind::i8 MMAs with both operands in shared memory.
qr_status launch_w8a8_gemm(const GemmJob& job, cudaStream_t stream);
// Packed e2m1 codes (two per byte, rows of K_p / 2 bytes): the same pair
// kernel with kind::f8f6f4 MMAs and an fp32 accumulator (acc_debug is then
// a float array).
qr_status launch_fp4_gemm(const GemmJob& job, cudaStream_t stream);

// M > 64: 2-SM tcgen05 MMA with the activation operand in TMEM, fp16
// outlier columns as a second MMA.
qr_status launch_w4a4_gemm_pair(const GemmJob& job, cudaStream_t stream);
// M <= 64: weights in TMEM, K split over a cluster.
qr_status launch_w4a4_gemm_decode(const GemmJob& job, cudaStream_t stream);
int decode_k_split(int64_t tiles, int64_t steps, int sms);
// The decode step in one kernel: the token rows of `rows` (M <= 64, a
// Hadamard, GSR or identity rotation) rotated and quantized into its codes,
// scales and outlier copy, then the decode GEMM on them, the two phases
// separated by a grid-wide barrier on the two words at `sync`.
qr_status launch_w4a4_decode_fused(const GemmJob& job, const RowJob& rows, uint32_t* sync,
                                   cudaStream_t stream);
int pair_tile_width(int64_t M, int64_t N, int sms);

// Row-major 2-D tensor map: `rows` rows of `cols` elements, row pitch
// `pitch_bytes`, box of box_cols x box_rows elements.
bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr,
                        uint64_t cols, uint64_t rows, uint64_t pitch_bytes, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swz);

qr_status launch_select_outliers(const uint16_t* x, int64_t T, int64_t K, int64_t ld,
                                 int32_t k, int32_t* idx_out, cudaStream_t stream);

// R3 on query rows: `vectors` contiguous head vectors of head_dim (32, 64,
// 128 or 256) fp16 values, each times H_d / sqrt(d), written as fp16.
qr_status launch_head_rotate(const uint16_t* src, uint16_t* dst, int64_t vectors, int head_dim,
                             cudaStream_t stream);

// KV-cache codes: `groups` rows of `group` (128 or 256) contiguous fp16
// values, each quantized asymmetrically to 4 bits (codes q - 8 packed two per
// byte, scale and zero point per row), R3 (Hadamard of head_dim, a power of
// two dividing the group) applied first when `rotate`.
qr_status launch_kv_group_quant(const uint16_t* src, int64_t groups, int group, int head_dim,
                                bool rotate, uint8_t* codes, float* scales, int32_t* zeros,
                                cudaStream_t stream);

qr_status launch_code_row_sums(const uint8_t* codes, int64_t rows, int64_t kp, int32_t* sums,
                               cudaStream_t stream);

// One thread waits, with the given limit, on an mbarrier nothing arrives on.
qr_status launch_wait_selfcheck(uint64_t limit_ns, cudaStream_t stream);

qr_status launch_invert_transpose(const float* P, int32_t n, float* out, int32_t* info,
                                  cudaStream_t stream);

}  // namespace qr
