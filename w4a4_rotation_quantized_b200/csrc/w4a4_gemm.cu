// w4a4_gemm.cu -- the W4A4 linear on fifth-generation tensor cores.
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
// Warp roles (320 threads, one CTA per SM, persistent over tiles):
//   warps 0-3  epilogue: TMEM -> registers, dequant, + outlier product, fp16 store
//   warps 4-7  widen:    packed stage (smem) -> 8-bit canonical SW128 stage (smem)
//   warp  8    producer: TMA loads of packed tiles and fp16 outlier tiles
//   warp  9    MMA:      TMEM allocation; one thread issues tcgen05.mma
// Tiles are 128 (MMA M, = TMEM lanes) x BN (MMA N).  The accumulator is
// double-buffered in TMEM so the epilogue of one tile overlaps the MMAs of
// the next.  For decode-sized M (<= 64) the kernel runs "swapped": weight rows
// take the MMA M side and tokens the N side (Y^T = W X^T).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

constexpr int kBM = 128;          // tile rows on the MMA M side
constexpr int kStepBytes = 64;    // packed bytes per row per K step (128 codes)
constexpr int kNP = 4;            // packed ring depth
constexpr int kNW = 2;            // widened ring depth
constexpr int kNO = 2;            // outlier ring depth
constexpr int kOutStep = 32;      // fp16 outlier columns per step (64-byte rows)
constexpr int kThreads = 320;
constexpr int kWidenThreads = 128;

struct GemmParams {
  const float* scale_a;   // per MMA-M row (normal: a_scales, swapped: w_scales)
  const float* scale_b;   // per MMA-N row
  __half* Y;
  int64_t ldy;
  int32_t* acc_debug;     // [M x N] or null
  int32_t rows_a, rows_b; // MMA-M-side and MMA-N-side row counts
  int32_t kt, ot;         // int4 K steps, outlier steps
  int32_t tiles_a, tiles_b;
  int32_t y_vec_ok;       // 16-byte fp16 stores allowed along n
  int32_t M, N;           // output shape (acc_debug row stride N)
  int32_t* status;
};

template <int BN, bool OUT>
struct Smem {
  static constexpr int kPackA = kBM * kStepBytes;          // 8 KB
  static constexpr int kPackB = BN * kStepBytes;
  static constexpr int kWideA = kBM * 2 * kStepBytes;      // 16 KB
  static constexpr int kWideB = BN * 2 * kStepBytes;
  static constexpr int kOutA = OUT ? kBM * kOutStep * 2 : 0;   // 8 KB
  static constexpr int kOutB = OUT ? BN * kOutStep * 2 : 0;
  static constexpr int off_wide_a = 0;                                  // 1024-aligned
  static constexpr int off_wide_b = off_wide_a + kNW * kWideA;
  static constexpr int off_out_a = off_wide_b + kNW * kWideB;
  static constexpr int off_out_b = off_out_a + kNO * kOutA;
  static constexpr int off_pack_a = off_out_b + kNO * kOutB;
  static constexpr int off_pack_b = off_pack_a + kNP * kPackA;
  static constexpr int off_bar = off_pack_b + kNP * kPackB;
  // barriers: full_p, empty_p, full_w, empty_w, full_o, empty_o (per slot),
  // tmem_full[2], tmem_empty[2], drain
  static constexpr int kNumBars = 2 * kNP + 2 * kNW + 2 * kNO + 5;
  static constexpr int off_misc = off_bar + 8 * kNumBars;
  static constexpr int kBytes = off_misc + 16 + 1024;    // + slack for 1024 alignment
};

template <int BN, bool SWAP, bool OUT>
__global__ void __launch_bounds__(kThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const __grid_constant__ CUtensorMap map_oa, const __grid_constant__ CUtensorMap map_ob,
                 const GemmParams p) {
  using S = Smem<BN, OUT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::off_bar);
  uint64_t* full_p = bars;
  uint64_t* empty_p = full_p + kNP;
  uint64_t* full_w = empty_p + kNP;
  uint64_t* empty_w = full_w + kNW;
  uint64_t* full_o = empty_w + kNW;
  uint64_t* empty_o = full_o + kNO;
  uint64_t* tmem_full = empty_o + kNO;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::off_misc);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + S::off_misc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kColsPerBuf = OUT ? 2 * BN : BN;
  constexpr uint32_t kTmemCols = (2 * kColsPerBuf <= 32) ? 32 : (2 * kColsPerBuf <= 64) ? 64
                                 : (2 * kColsPerBuf <= 128) ? 128 : (2 * kColsPerBuf <= 256) ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNP; ++i) { mbar_init(&full_p[i], 1); mbar_init(&empty_p[i], 4); }
    for (int i = 0; i < kNW; ++i) { mbar_init(&full_w[i], 4); mbar_init(&empty_w[i], 1); }
    for (int i = 0; i < kNO; ++i) { mbar_init(&full_o[i], 1); mbar_init(&empty_o[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tmem_full[i], 1); mbar_init(&tmem_empty[i], 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    if (p.kt > 0) { tma_prefetch_desc(&map_a); tma_prefetch_desc(&map_b); }
    if (OUT && p.ot > 0) { tma_prefetch_desc(&map_oa); tma_prefetch_desc(&map_ob); }
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.tiles_a * p.tiles_b;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0, ot = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int ta = tile % p.tiles_a, tb = tile / p.tiles_a;
        for (int ks = 0; ks < p.kt && ok; ++ks, ++it) {
          const uint32_t s = it % kNP, ph = (it / kNP) & 1;
          if (!(ok = mbar_wait_bounded(&empty_p[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
          mbar_arrive_expect_tx(&full_p[s], S::kPackA + S::kPackB);
          tma_load_2d(smem + S::off_pack_a + s * S::kPackA, &map_a, &full_p[s], ks * kStepBytes, ta * kBM);
          tma_load_2d(smem + S::off_pack_b + s * S::kPackB, &map_b, &full_p[s], ks * kStepBytes, tb * BN);
        }
        if (OUT) {
          for (int os = 0; os < p.ot && ok; ++os, ++ot) {
            const uint32_t s = ot % kNO, ph = (ot / kNO) & 1;
            if (!(ok = mbar_wait_bounded(&empty_o[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
            mbar_arrive_expect_tx(&full_o[s], S::kOutA + S::kOutB);
            tma_load_2d(smem + S::off_out_a + s * S::kOutA, &map_oa, &full_o[s], os * kOutStep, ta * kBM);
            tma_load_2d(smem + S::off_out_b + s * S::kOutB, &map_ob, &full_o[s], os * kOutStep, tb * BN);
          }
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA's shared memory
        // goes away.
        for (uint32_t i = (it > kNP ? it - kNP : 0); i < it; ++i)
          mbar_wait_bounded(&full_p[i % kNP], (i / kNP) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
        for (uint32_t i = (ot > kNO ? ot - kNO : 0); i < ot; ++i)
          mbar_wait_bounded(&full_o[i % kNO], (i / kNO) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BN);
      constexpr uint32_t idesc_o = idesc_f16(BN);
      uint32_t wi = 0, ot = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
        if (!(ok = mbar_wait_bounded(&tmem_empty[buf], tph ^ 1, abort_flag, p.status, kDevTimeoutMma))) break;
        tc_fence_after();
        const uint32_t d_int = tmem_base + buf * kColsPerBuf;
        for (int ks = 0; ks < p.kt; ++ks, ++wi) {
          const uint32_t s = wi % kNW, ph = (wi / kNW) & 1;
          if (!(ok = mbar_wait_bounded(&full_w[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          tc_fence_after();
          const uint64_t da = smem_desc_kmajor(smem_u32(smem + S::off_wide_a + s * S::kWideA), 128);
          const uint64_t db = smem_desc_kmajor(smem_u32(smem + S::off_wide_b + s * S::kWideB), 128);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8(d_int, da + 2 * k, db + 2 * k, idesc, (ks | k) != 0);
          mma_commit(&empty_w[s]);
        }
        if (OUT && ok) {
          const uint32_t d_out = d_int + BN;
          for (int os = 0; os < p.ot; ++os, ++ot) {
            const uint32_t s = ot % kNO, ph = (ot / kNO) & 1;
            if (!(ok = mbar_wait_bounded(&full_o[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
            tc_fence_after();
            const uint64_t da = smem_desc_kmajor(smem_u32(smem + S::off_out_a + s * S::kOutA), 64);
            const uint64_t db = smem_desc_kmajor(smem_u32(smem + S::off_out_b + s * S::kOutB), 64);
#pragma unroll
            for (int k = 0; k < 2; ++k)
              mma_f16(d_out, da + 2 * k, db + 2 * k, idesc_o, (os | k) != 0);
            mma_commit(&empty_o[s]);
          }
        }
        if (ok) mma_commit(&tmem_full[buf]);
      }
      // Every MMA issued must finish before tensor memory is released.
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, abort_flag, p.status, kDevTimeoutDrain, kDrainLimitNs);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ widen
    const int wt = threadIdx.x - 128;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int ks = 0; ks < p.kt; ++ks, ++it) {
        const uint32_t s = it % kNP, ph = (it / kNP) & 1;
        const uint32_t sw = it % kNW, phw = (it / kNW) & 1;
        if (!(ok = mbar_wait_bounded(&full_p[s], ph, abort_flag, p.status, kDevTimeoutWiden))) break;
        if (!(ok = mbar_wait_bounded(&empty_w[sw], phw ^ 1, abort_flag, p.status, kDevTimeoutWiden))) break;
        const uint8_t* pa = smem + S::off_pack_a + s * S::kPackA;
        const uint8_t* pb = smem + S::off_pack_b + s * S::kPackB;
        uint8_t* wa = smem + S::off_wide_a + sw * S::kWideA;
        uint8_t* wb = smem + S::off_wide_b + sw * S::kWideB;
        constexpr int kTasks = (kBM + BN) * 4;    // 16-byte packed chunks
#pragma unroll 4
        for (int task = wt; task < kTasks; task += kWidenThreads) {
          const int row = task >> 2, c = task & 3;
          const bool is_a = row < kBM;
          const int r = is_a ? row : row - kBM;
          const uint4 u = *reinterpret_cast<const uint4*>((is_a ? pa : pb) + r * kStepBytes + c * 16);
          uint4 ev, od;
          ev.x = (u.x << 4) & 0xF0F0F0F0u; od.x = u.x & 0xF0F0F0F0u;
          ev.y = (u.y << 4) & 0xF0F0F0F0u; od.y = u.y & 0xF0F0F0F0u;
          ev.z = (u.z << 4) & 0xF0F0F0F0u; od.z = u.z & 0xF0F0F0F0u;
          ev.w = (u.w << 4) & 0xF0F0F0F0u; od.w = u.w & 0xF0F0F0F0u;
          uint8_t* base = (is_a ? wa : wb) + (r >> 3) * 1024 + (r & 7) * 128;
          *reinterpret_cast<uint4*>(base + (((2 * c) ^ (r & 7)) << 4)) = ev;
          *reinterpret_cast<uint4*>(base + (((2 * c + 1) ^ (r & 7)) << 4)) = od;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full_w[sw]);
          mbar_arrive(&empty_p[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int lrow = warp * 32 + lane;            // TMEM lane = tile row
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    uint32_t tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
      const int ta = tile % p.tiles_a, tb = tile / p.tiles_a;
      const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
      if (!(ok = mbar_wait_bounded(&tmem_full[buf], tph, abort_flag, p.status, kDevTimeoutEpilogue))) break;
      tc_fence_after();
      const int ra = ta * kBM + lrow;             // MMA-M row (m, or n when swapped)
      const bool ra_ok = ra < p.rows_a;
      const float s_row = ra_ok ? __ldg(p.scale_a + ra) * (1.0f / 256.0f) : 0.0f;
      const uint32_t t_int = tmem_base + lane_off + buf * kColsPerBuf;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t acc[32];
        uint32_t oacc[32];
        tmem_ld_32x32b_x32(t_int + c * 32, acc);
        if (OUT) tmem_ld_32x32b_x32(t_int + BN + c * 32, oacc);
        tmem_ld_wait();
        if (p.kt == 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[j] = 0;
        }
        if (OUT && p.ot == 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j) oacc[j] = 0;
        }
        const int cb0 = tb * BN + c * 32;          // first MMA-N row of this chunk
        if (!ra_ok) continue;
        if (!SWAP) {
          // lane owns output row m = ra; columns n = cb0 + j
          const int m = ra;
          uint32_t hp[16];                         // 32 fp16, two per word
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float y2[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int n = cb0 + j + t;
              const float sb = (n < p.rows_b) ? __ldg(p.scale_b + n) : 0.0f;
              y2[t] = static_cast<float>(static_cast<int32_t>(acc[j + t])) * s_row * sb;
              if (OUT) y2[t] += __uint_as_float(oacc[j + t]);
            }
            const __half2 h2 = __floats2half2_rn(y2[0], y2[1]);
            hp[j / 2] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          __half* yrow = p.Y + static_cast<int64_t>(m) * p.ldy;
          if (p.y_vec_ok && cb0 + 32 <= p.rows_b) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(yrow + cb0 + 8 * q) =
                  make_uint4(hp[4 * q], hp[4 * q + 1], hp[4 * q + 2], hp[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (cb0 + j < p.rows_b) {
                const uint16_t bits = static_cast<uint16_t>(hp[j / 2] >> (16 * (j & 1)));
                reinterpret_cast<uint16_t*>(yrow)[cb0 + j] = bits;
              }
            }
          }
          if (p.acc_debug != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (cb0 + j < p.rows_b)
                p.acc_debug[static_cast<int64_t>(m) * p.N + cb0 + j] = static_cast<int32_t>(acc[j]) >> 8;
          }
        } else {
          // lane owns output column n = ra; rows m = cb0 + j (tokens)
          const int n = ra;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = cb0 + j;
            if (m >= p.rows_b) continue;
            float y = static_cast<float>(static_cast<int32_t>(acc[j])) * s_row * __ldg(p.scale_b + m);
            if (OUT) y += __uint_as_float(oacc[j]);
            p.Y[static_cast<int64_t>(m) * p.ldy + n] = __float2half_rn(y);
            if (p.acc_debug != nullptr)
              p.acc_debug[static_cast<int64_t>(m) * p.N + n] = static_cast<int32_t>(acc[j]) >> 8;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

// ------------------------------------------------------------------ host side

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
  return fn(map, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int BN, bool SWAP, bool OUT>
cudaError_t run(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& moa,
                const CUtensorMap& mob, const GemmParams& p, cudaStream_t stream) {
  auto k = w4a4_gemm_kernel<BN, SWAP, OUT>;
  const int smem = Smem<BN, OUT>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.tiles_a * p.tiles_b, sm_count());
  k<<<grid, kThreads, smem, stream>>>(ma, mb, moa, mob, p);
  return cudaGetLastError();
}

template <bool SWAP, bool OUT>
cudaError_t run_bn(int bn, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& moa,
                   const CUtensorMap& mob, const GemmParams& p, cudaStream_t s) {
  switch (bn) {
    case 32: return run<32, SWAP, OUT>(ma, mb, moa, mob, p, s);
    case 64: return run<64, SWAP, OUT>(ma, mb, moa, mob, p, s);
    case 128: return run<128, SWAP, OUT>(ma, mb, moa, mob, p, s);
    default: return run<256, SWAP, OUT && false>(ma, mb, moa, mob, p, s);
  }
}

}  // namespace

qr_status launch_w4a4_gemm(const GemmJob& j, cudaStream_t stream) {
  if (j.M == 0 || j.N == 0) return QR_OK;
  return launch_w4a4_gemm_pair(j, stream);
}

qr_status launch_w4a4_gemm_single(const GemmJob& j, cudaStream_t stream) {
  if (j.M == 0 || j.N == 0) return QR_OK;
  const bool swap = j.M <= 64;
  const bool out = j.n_out > 0;
  const int64_t rows_a = swap ? j.N : j.M;      // MMA-M side
  const int64_t rows_b = swap ? j.M : j.N;      // MMA-N side
  int bn;
  if (swap) {
    bn = 32;
    while (bn < rows_b) bn *= 2;                 // 32, 64
  } else {
    bn = out ? 128 : 256;
  }
  const uint8_t* ca = swap ? j.w_codes : j.a_codes;
  const uint8_t* cb = swap ? j.a_codes : j.w_codes;
  const uint16_t* oa = swap ? j.w_out : j.x_out;
  const uint16_t* ob = swap ? j.x_out : j.w_out;

  GemmParams p{};
  p.scale_a = swap ? j.w_scales : j.a_scales;
  p.scale_b = swap ? j.a_scales : j.w_scales;
  p.Y = reinterpret_cast<__half*>(j.Y);
  p.ldy = j.ldy;
  p.acc_debug = j.acc_debug;
  p.rows_a = static_cast<int32_t>(rows_a);
  p.rows_b = static_cast<int32_t>(rows_b);
  p.kt = static_cast<int32_t>(j.Kp / 128);
  p.ot = out ? (j.n_out + kOutStep - 1) / kOutStep : 0;
  p.tiles_a = static_cast<int32_t>((rows_a + kBM - 1) / kBM);
  p.tiles_b = static_cast<int32_t>((rows_b + bn - 1) / bn);
  p.y_vec_ok = (reinterpret_cast<uintptr_t>(j.Y) % 16 == 0) && (j.ldy % 8 == 0);
  p.M = static_cast<int32_t>(j.M);
  p.N = static_cast<int32_t>(j.N);
  p.status = device_status_word();
  if (p.status == nullptr) return QR_ERR_CUDA;

  CUtensorMap ma{}, mb{}, moa{}, mob{};
  const uint64_t kb = static_cast<uint64_t>(j.Kp) / 2;   // packed bytes per row
  if (p.kt > 0 &&
      (!make_tensor_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, ca, kb, rows_a, kb, kStepBytes, kBM,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
       !make_tensor_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, cb, kb, rows_b, kb, kStepBytes, bn,
                 CU_TENSOR_MAP_SWIZZLE_NONE)))
    return QR_ERR_CUDA;
  if (out) {
    const uint64_t no = static_cast<uint64_t>(j.n_out);
    if (!make_tensor_map_2d(&moa, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, oa, no, rows_a, no * 2, kOutStep, kBM,
                  CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_tensor_map_2d(&mob, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ob, no, rows_b, no * 2, kOutStep, bn,
                  CU_TENSOR_MAP_SWIZZLE_64B))
      return QR_ERR_CUDA;
  } else {
    moa = ma;
    mob = mb;
  }
  cudaError_t e;
  if (swap) e = out ? run_bn<true, true>(bn, ma, mb, moa, mob, p, stream)
                    : run_bn<true, false>(bn, ma, mb, moa, mob, p, stream);
  else e = out ? run_bn<false, true>(bn, ma, mb, moa, mob, p, stream)
               : run_bn<false, false>(bn, ma, mb, moa, mob, p, stream);
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
