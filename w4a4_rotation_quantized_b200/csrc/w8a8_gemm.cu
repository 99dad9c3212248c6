// w8a8_gemm.cu -- the 8-bit linear of QUIK's INT8 layers.
//
// "QUIK：LLM上的一种4-bit推理方法", QUIK量化 results: the LLaMA-2 down_proj
// stays in INT8 with more outlier columns, and QUIK-8B runs every layer in
// INT8.  Same computation as the W4A4 linear, with 8-bit codes:
//
//   acc[m, n] = sum_k qa[m, k] qw[n, k]                 (exact int32)
//   Y[m, n]   = fp16(acc * sa[m] * sw[n] + sum_j x_out[m, j] w_out[n, j])
//
// 8-bit codes are the tcgen05 kind::i8 operands as they are, so there is no
// widening step: TMA stages both packed tiles straight into the canonical
// 128-byte-swizzled K-major layout and one thread issues the MMAs with both
// operands in shared memory.  A K step is 128 codes (a 128-byte row); the
// fp16 outlier columns, 64 per step (also 128-byte rows), ride the same ring
// as extra steps whose MMAs (kind::f16) go to an fp32 accumulator.
//
// Ring: six stages at BN = 128 (32 KB each), four at BN = 256 (48 KB).
// Tile: 128 activation rows x BN weight rows, persistent over tiles with the
// activation tiles fastest (concurrent CTAs share a weight tile in L2).
// Tensor memory: two accumulator buffers (the epilogue of one tile overlaps
// the next tile's MMAs), each BN int32 columns plus BN fp32 outlier columns
// when there are outliers.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM allocation and
// the MMA-issuing thread, warps 2-5 epilogue (thread = TMEM lane = output
// row).  Every wait is bounded.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

constexpr int kRow = 128;            // bytes per row per step (128 int8 or 64 fp16)
constexpr int kThreads8 = 192;

template <int BN>
struct W8Smem {
  // ring depth: about 190 KB of stages (4 at BN = 256, 6 at BN = 128), so
  // that the loads in flight cover the memory latency at the MMA rate
  static constexpr int kStages = BN >= 256 ? 4 : 6;
  static constexpr int kA = 128 * kRow;                    // 16 KB
  static constexpr int kB = BN * kRow;
  static constexpr int kStage = kA + kB;
  static constexpr int off_ring = 0;
  static constexpr int off_sb = off_ring + kStages * kStage;    // per warp: the tile's weight scales
  static constexpr int off_bar = off_sb + 4 * BN * 4;
  // full[stages], empty[stages], tmem_full[2], tmem_empty[2], drain
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int off_misc = off_bar + 8 * kNumBars;
  static constexpr int kBytes = off_misc + 16 + 1024;
  static_assert(kStage % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

struct W8Params {
  const float* a_scales;
  const float* w_scales;
  __half* Y;
  int64_t ldy;
  int32_t* acc_debug;
  int32_t M, N;
  int32_t kt, ot;                  // int8 K steps, outlier steps
  int32_t tiles_m, tiles_n;
  int32_t y_vec_ok;
  int32_t* status;
};

template <int BN, bool OUT>
__global__ void __launch_bounds__(kThreads8, 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const __grid_constant__ CUtensorMap map_oa,
                 const __grid_constant__ CUtensorMap map_ob, const W8Params p) {
  using S = W8Smem<BN>;
  constexpr int kStages = S::kStages;
  constexpr uint32_t kColsAcc = OUT ? 2 * BN : BN;
  static_assert(2 * kColsAcc <= 512, "tensor memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::off_bar);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* tmem_full = empty + kStages;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::off_misc);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + S::off_misc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tmem_full[i], 1);
      mbar_init(&tmem_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    if (p.kt > 0) { tma_prefetch_desc(&map_a); tma_prefetch_desc(&map_b); }
    if (OUT && p.ot > 0) { tma_prefetch_desc(&map_oa); tma_prefetch_desc(&map_ob); }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();
  grid_dep_launch();

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int steps = p.kt + (OUT ? p.ot : 0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int ym = (tile % p.tiles_m) * 128, yn = (tile / p.tiles_m) * BN;
        for (int st = 0; st < steps; ++st, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
          mbar_arrive_expect_tx(&full[s], S::kStage);
          uint8_t* sa = smem + S::off_ring + s * S::kStage;
          if (st < p.kt) {
            tma_load_2d(sa, &map_a, &full[s], st * kRow, ym);
            tma_load_2d(sa + S::kA, &map_b, &full[s], st * kRow, yn);
          } else {
            const int os = st - p.kt;
            tma_load_2d(sa, &map_oa, &full[s], os * (kRow / 2), ym);
            tma_load_2d(sa + S::kA, &map_ob, &full[s], os * (kRow / 2), yn);
          }
        }
      }
      if (!ok)
        for (uint32_t i = (it > kStages ? it - kStages : 0); i < it; ++i)
          mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BN);
      constexpr uint32_t idesc_o = idesc_f16(BN);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
        if (!(ok = mbar_wait_bounded(&tmem_empty[buf], tph ^ 1, abort_flag, p.status, kDevTimeoutMma))) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * kColsAcc;
        for (int st = 0; st < steps; ++st, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait_bounded(&full[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + S::off_ring + s * S::kStage);
          const uint64_t da = smem_desc_kmajor(sa, 128), db = smem_desc_kmajor(sa + S::kA, 128);
          if (st < p.kt) {
#pragma unroll
            for (int k = 0; k < 4; ++k)       // 4 x K32 (32 bytes each)
              mma_i8(d, da + 2 * k, db + 2 * k, idesc, (st | k) != 0);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)       // 4 x K16 fp16 (32 bytes each)
              mma_f16(d + BN, da + 2 * k, db + 2 * k, idesc_o, ((st - p.kt) | k) != 0);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&tmem_full[buf]);
      }
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, abort_flag, p.status, kDevTimeoutDrain, kDrainLimitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                        // TMEM lane quadrant
    const int lrow = 32 * q + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    float* sb = reinterpret_cast<float*>(smem + S::off_sb) + (warp - 2) * BN;
    uint32_t tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
      __syncwarp();
      for (int i = lane; i < BN; i += 32) {
        const int n = tn * BN + i;
        sb[i] = n < p.N ? __ldg(p.w_scales + n) : 0.0f;
      }
      __syncwarp();
      if (!(ok = mbar_wait_bounded(&tmem_full[buf], tph, abort_flag, p.status, kDevTimeoutEpilogue))) break;
      tc_fence_after();
      const int m = tm * 128 + lrow;
      const bool m_ok = m < p.M;
      const float sa = m_ok ? __ldg(p.a_scales + m) : 0.0f;
      const uint32_t t_acc = tmem + lane_off + buf * kColsAcc;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t acc[32], oacc[32];
        tmem_ld_32x32b_x32(t_acc + 32 * c, acc);
        if (OUT) tmem_ld_32x32b_x32(t_acc + BN + 32 * c, oacc);
        tmem_ld_wait();
        const bool kz = p.kt == 0, oz = OUT && p.ot == 0;
        const int n0 = tn * BN + 32 * c;
        uint32_t hp[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float y0 = kz ? 0.0f : static_cast<float>(static_cast<int32_t>(acc[2 * j])) * sa * sb[32 * c + 2 * j];
          float y1 = kz ? 0.0f : static_cast<float>(static_cast<int32_t>(acc[2 * j + 1])) * sa * sb[32 * c + 2 * j + 1];
          if (OUT && !oz) {
            y0 += __uint_as_float(oacc[2 * j]);
            y1 += __uint_as_float(oacc[2 * j + 1]);
          }
          const __half2 h = __floats2half2_rn(y0, y1);
          hp[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        if (m_ok) {
          __half* yrow = p.Y + static_cast<int64_t>(m) * p.ldy;
          if (p.y_vec_ok && n0 + 32 <= p.N) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              *reinterpret_cast<uint4*>(yrow + n0 + 8 * v) =
                  make_uint4(hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < p.N)
                reinterpret_cast<uint16_t*>(yrow)[n0 + j] = static_cast<uint16_t>(hp[j / 2] >> (16 * (j & 1)));
          }
          if (p.acc_debug != nullptr)
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < p.N)
                p.acc_debug[static_cast<int64_t>(m) * p.N + n0 + j] = kz ? 0 : static_cast<int32_t>(acc[j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int BN, bool OUT>
cudaError_t run_w8(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& moa,
                   const CUtensorMap& mob, const W8Params& p, cudaStream_t stream) {
  auto k = w8a8_gemm_kernel<BN, OUT>;
  const int smem = W8Smem<BN>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.tiles_m * p.tiles_n, sm_count());
  e = launch_pdl(k, dim3(grid), dim3(kThreads8), smem, stream, 1, ma, mb, moa, mob, p);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace

qr_status launch_w8a8_gemm(const GemmJob& j, cudaStream_t stream) {
  if (j.M == 0 || j.N == 0) return QR_OK;
  const bool out = j.n_out > 0;
  W8Params p{};
  p.a_scales = j.a_scales;
  p.w_scales = j.w_scales;
  p.Y = reinterpret_cast<__half*>(j.Y);
  p.ldy = j.ldy;
  p.acc_debug = j.acc_debug;
  p.M = static_cast<int32_t>(j.M);
  p.N = static_cast<int32_t>(j.N);
  p.kt = static_cast<int32_t>(j.Kp / kRow);
  p.ot = out ? (j.n_out + kRow / 2 - 1) / (kRow / 2) : 0;
  const int bn = out ? 128 : 256;
  p.tiles_m = static_cast<int32_t>((j.M + 127) / 128);
  p.tiles_n = static_cast<int32_t>((j.N + bn - 1) / bn);
  p.y_vec_ok = (reinterpret_cast<uintptr_t>(j.Y) % 16 == 0) && (j.ldy % 8 == 0);
  p.status = device_status_word();
  if (p.status == nullptr) return QR_ERR_CUDA;
  CUtensorMap ma{}, mb{}, moa{}, mob{};
  const uint64_t kb = static_cast<uint64_t>(j.Kp);        // one byte per code
  if (p.kt > 0 &&
      (!make_tensor_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.a_codes, kb, j.M, kb, kRow, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
       !make_tensor_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.w_codes, kb, j.N, kb, kRow, bn,
                           CU_TENSOR_MAP_SWIZZLE_128B)))
    return QR_ERR_CUDA;
  if (out) {
    const uint64_t no = static_cast<uint64_t>(j.n_out);
    if (!make_tensor_map_2d(&moa, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.x_out, no, j.M, no * 2,
                            kRow / 2, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tensor_map_2d(&mob, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.w_out, no, j.N, no * 2,
                            kRow / 2, bn, CU_TENSOR_MAP_SWIZZLE_128B))
      return QR_ERR_CUDA;
  }
  const cudaError_t e = out ? run_w8<128, true>(ma, mb, moa, mob, p, stream)
                            : run_w8<256, false>(ma, mb, moa, mob, p, stream);
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
