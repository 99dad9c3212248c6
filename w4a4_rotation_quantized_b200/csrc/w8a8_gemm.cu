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
// widening step: TMA stages the code tiles straight into the canonical
// 128-byte-swizzled K-major layout and one thread issues the MMAs with both
// operands in shared memory.  A K step is 128 codes (a 128-byte row); the
// fp16 outlier columns, 64 per step (also 128-byte rows), ride the same ring
// as extra steps whose MMAs (kind::f16) go to an fp32 accumulator.
//
// The two CTAs of a cluster compute a 256 x 256 tile with
// tcgen05.mma.cta_group::2: each CTA stages its own 128 activation rows and
// half of the 256 weight rows, and the pair's MMA reads both halves.  Every
// operand byte staged in shared memory then feeds 256 x 128 MACs per K code,
// twice the single-CTA 128 x 256 tile's reuse, which halves the L2 -> SM
// traffic per MAC (the loop is bound by it otherwise).
//
// Ring: six stages of 32 KB per CTA.  Tiles are persistent over the CTA
// pairs, activation tiles fastest (concurrent pairs share a weight tile in
// L2).  Tensor memory per CTA: 256 int32 accumulator columns, plus 256 fp32
// outlier columns when there are outliers; without outliers two buffers
// alternate so that the epilogue of one tile overlaps the next tile's MMAs.
//
// Warp roles (192 threads per CTA): warp 0 TMA producer; warp 1 TMEM
// allocation and, in the even CTA, the MMA-issuing thread, in the odd CTA
// the thread that relays "stage landed" to the even CTA; warps 2-5 epilogue
// (thread = TMEM lane = output row).  Every wait is bounded.
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
constexpr int kBN8 = 256;            // weight rows per pair tile
constexpr int kHalf8 = kBN8 / 2;     // weight rows per CTA

struct W8Smem {
  static constexpr int kStages = 6;
  static constexpr int kA = 128 * kRow;                    // 16 KB
  static constexpr int kB = kHalf8 * kRow;                 // 16 KB
  static constexpr int kStage = kA + kB;
  static constexpr int off_ring = 0;
  static constexpr int off_sb = off_ring + kStages * kStage;    // per warp: the tile's weight scales
  static constexpr int off_bar = off_sb + 4 * kBN8 * 4;
  // full[stages], empty[stages], tmem_full[2], tmem_empty[2], drain
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int off_misc = off_bar + 8 * kNumBars;
  static constexpr int kBytes = off_misc + 16 + 1024;
  static_assert(kStage % 1024 == 0 && kA % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

struct W8Params {
  const float* a_scales;
  const float* w_scales;
  __half* Y;
  int64_t ldy;
  void* acc_debug;                 // int32 (8-bit codes) or float (e2m1 codes) [M x N], or null
  int32_t M, N;
  int32_t kt, ot;                  // int8 K steps, outlier steps
  int32_t tiles_m, tiles_n;        // 256-row activation tiles, 256-row weight tiles
  int32_t y_vec_ok;
  int32_t* status;
};

// FP4: e2m1 codes (kind::f8f6f4, fp32 accumulator), else 8-bit integer codes
// (kind::i8, int32 accumulator).  Both stage 128 codes per 128-byte row.
template <bool OUT, bool FP4>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads8, 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const __grid_constant__ CUtensorMap map_oa,
                 const __grid_constant__ CUtensorMap map_ob, const W8Params p) {
  using S = W8Smem;
  constexpr int kStages = S::kStages;
  constexpr int BN = kBN8;
  constexpr uint32_t kColsAcc = OUT ? 2 * BN : BN;
  constexpr uint32_t kNB = 512 / kColsAcc;                 // accumulator buffers
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::off_bar);
  uint64_t* full = bars;                   // local TMA landed (+ the odd CTA's relay, even CTA)
  uint64_t* empty = full + kStages;        // each CTA: the pair's MMAs are done with the stage
  uint64_t* tmem_full = empty + kStages;   // each CTA: accumulator ready
  uint64_t* tmem_empty = tmem_full + 2;    // even CTA: both epilogues drained (8 warps)
  uint64_t* drain = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::off_misc);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + S::off_misc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], leader ? 2 : 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tmem_full[i], 1);
      mbar_init(&tmem_empty[i], 8);
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
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                          // barriers of both CTAs initialized
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();
  grid_dep_launch();

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int steps = p.kt + (OUT ? p.ot : 0);
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
        const int ya = (tile % p.tiles_m) * 256 + static_cast<int>(rank) * 128;
        const int yb = (tile / p.tiles_m) * BN + static_cast<int>(rank) * kHalf8;
        for (int st = 0; st < steps; ++st, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait_cluster_bounded(&empty[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
          // e2m1 tiles count the packed bytes read (half the 128-byte rows
          // they fill in shared memory)
          mbar_arrive_expect_tx(&full[s], (FP4 && st < p.kt) ? S::kStage / 2 : S::kStage);
          uint8_t* sa = smem + S::off_ring + s * S::kStage;
          if (st < p.kt) {
            tma_load_2d(sa, &map_a, &full[s], st * kRow, ya);
            tma_load_2d(sa + S::kA, &map_b, &full[s], st * kRow, yb);
          } else {
            const int os = st - p.kt;
            tma_load_2d(sa, &map_oa, &full[s], os * (kRow / 2), ya);
            tma_load_2d(sa + S::kA, &map_ob, &full[s], os * (kRow / 2), yb);
          }
        }
      }
      if (!ok)
        for (uint32_t i = (it > kStages ? it - kStages : 0); i < it; ++i)
          mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
    }
  } else if (warp == 1) {
    if (!leader && lane == 0) {
      // ------------------------------------------------------------ relay (odd CTA)
      // This CTA's stage landed -> the even CTA's full barrier.  The local
      // wait acquires the TMA's completion.
      const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl)
        for (int st = 0; st < steps; ++st, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait_bounded(&full[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          mbar_arrive_cluster_relaxed(full0 + s * 8);
        }
    }
    if (leader && lane == 0) {
      // ------------------------------------------------------------ MMA (even CTA)
      constexpr uint32_t idesc = FP4 ? idesc_e2m1_m256(BN) : idesc_i8_m256(BN);
      constexpr uint32_t idesc_o = idesc_f16_m256(BN);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++tcount) {
        const uint32_t buf = tcount % kNB, tph = (tcount / kNB) & 1;
        if (!(ok = mbar_wait_cluster_bounded(&tmem_empty[buf], tph ^ 1, abort_flag, p.status, kDevTimeoutMma))) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * kColsAcc;
        for (int st = 0; st < steps; ++st, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!(ok = mbar_wait_cluster_bounded(&full[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + S::off_ring + s * S::kStage);
          const uint64_t da = smem_desc_kmajor(sa, 128), db = smem_desc_kmajor(sa + S::kA, 128);
          if (st < p.kt) {
#pragma unroll
            for (int k = 0; k < 4; ++k)       // 4 x K32 (32 bytes each)
              if constexpr (FP4)
                mma_f8f6f4_pair(d, da + 2 * k, db + 2 * k, idesc, (st | k) != 0);
              else
                mma_i8_pair(d, da + 2 * k, db + 2 * k, idesc, (st | k) != 0);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)       // 4 x K16 fp16 (32 bytes each)
              mma_f16_pair(d + BN, da + 2 * k, db + 2 * k, idesc_o, ((st - p.kt) | k) != 0);
          }
          mma_commit_pair(&empty[s], 0x3);
        }
        if (ok) mma_commit_pair(&tmem_full[buf], 0x3);
      }
      mma_commit_pair_local(drain);
      mbar_wait_bounded(drain, 0, abort_flag, p.status, kDevTimeoutDrain, kDrainLimitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                        // TMEM lane quadrant
    const int lrow = 32 * q + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    float* sb = reinterpret_cast<float*>(smem + S::off_sb) + (warp - 2) * BN;
    const uint32_t tmem_empty0 = mapa_shared(smem_u32(&tmem_empty[0]), 0);
    uint32_t tcount = 0;
    bool ok = true;
    for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++tcount) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const uint32_t buf = tcount % kNB, tph = (tcount / kNB) & 1;
      __syncwarp();
      for (int i = lane; i < BN; i += 32) {
        const int n = tn * BN + i;
        sb[i] = n < p.N ? __ldg(p.w_scales + n) : 0.0f;
      }
      __syncwarp();
      if (!(ok = mbar_wait_cluster_bounded(&tmem_full[buf], tph, abort_flag, p.status, kDevTimeoutEpilogue))) break;
      tc_fence_after();
      const int m = tm * 256 + static_cast<int>(rank) * 128 + lrow;
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
          const float a0 = FP4 ? __uint_as_float(acc[2 * j]) : static_cast<float>(static_cast<int32_t>(acc[2 * j]));
          const float a1 = FP4 ? __uint_as_float(acc[2 * j + 1]) : static_cast<float>(static_cast<int32_t>(acc[2 * j + 1]));
          float y0 = kz ? 0.0f : a0 * sa * sb[32 * c + 2 * j];
          float y1 = kz ? 0.0f : a1 * sa * sb[32 * c + 2 * j + 1];
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
              if (n0 + j < p.N)          // raw accumulator bits: int32, or the fp32 sum
                static_cast<uint32_t*>(p.acc_debug)[static_cast<int64_t>(m) * p.N + n0 + j] = kz ? 0u : acc[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty0 + buf * 8);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                          // no CTA leaves while its pair may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

template <bool OUT, bool FP4>
cudaError_t run_w8(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& moa,
                   const CUtensorMap& mob, const W8Params& p, cudaStream_t stream) {
  auto k = w8a8_gemm_kernel<OUT, FP4>;
  const int smem = W8Smem::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int clusters = std::min(p.tiles_m * p.tiles_n, sm_count() / 2);
  e = launch_pdl(k, dim3(2 * clusters), dim3(kThreads8), smem, stream, 1, ma, mb, moa, mob, p);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace

// The pair kernel on 8-bit integer codes (one byte per code) or on packed
// e2m1 codes (two per byte), which TMA unpacks into the tensor core's
// 16-byte-aligned 4-bit layout (8 bytes of 16 codes, then 8 bytes of gap).
qr_status launch_pair_gemm8(const GemmJob& j, bool fp4, cudaStream_t stream) {
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
  p.tiles_m = static_cast<int32_t>((j.M + 255) / 256);
  p.tiles_n = static_cast<int32_t>((j.N + kBN8 - 1) / kBN8);
  p.y_vec_ok = (reinterpret_cast<uintptr_t>(j.Y) % 16 == 0) && (j.ldy % 8 == 0);
  p.status = device_status_word();
  if (p.status == nullptr) return QR_ERR_CUDA;
  CUtensorMap ma{}, mb{}, moa{}, mob{};
  if (p.kt > 0) {
    const uint64_t kc = static_cast<uint64_t>(j.Kp);                  // codes per row
    const uint64_t pitch = fp4 ? kc / 2 : kc;                          // bytes per row
    const CUtensorMapDataType dt = fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    if (!make_tensor_map_2d(&ma, dt, j.a_codes, kc, j.M, pitch, kRow, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tensor_map_2d(&mb, dt, j.w_codes, kc, j.N, pitch, kRow, kHalf8, CU_TENSOR_MAP_SWIZZLE_128B))
      return QR_ERR_CUDA;
  }
  if (out) {
    const uint64_t no = static_cast<uint64_t>(j.n_out);
    if (!make_tensor_map_2d(&moa, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.x_out, no, j.M, no * 2,
                            kRow / 2, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tensor_map_2d(&mob, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.w_out, no, j.N, no * 2,
                            kRow / 2, kHalf8, CU_TENSOR_MAP_SWIZZLE_128B))
      return QR_ERR_CUDA;
  }
  cudaError_t e;
  if (fp4)
    e = out ? run_w8<true, true>(ma, mb, moa, mob, p, stream) : run_w8<false, true>(ma, mb, moa, mob, p, stream);
  else
    e = out ? run_w8<true, false>(ma, mb, moa, mob, p, stream) : run_w8<false, false>(ma, mb, moa, mob, p, stream);
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

qr_status launch_w8a8_gemm(const GemmJob& j, cudaStream_t stream) {
  return launch_pair_gemm8(j, false, stream);
}

qr_status launch_fp4_gemm(const GemmJob& j, cudaStream_t stream) {
  return launch_pair_gemm8(j, true, stream);
}

}  // namespace qr
