// w4a4_gemm_pair.cu -- the W4A4 linear on a pair of SMs (prefill shapes).
//
// Same computation as w4a4_gemm.cu (QUIK §4: INT4 codes multiplied on
// integer tensor cores with INT32 accumulation, dequantized per token and
// per channel in the epilogue), arranged to move fewer bytes through shared
// memory per MMA:
//
//  * tcgen05.mma.cta_group::2: the two CTAs of a cluster compute a 256 x BN
//    tile; each CTA holds its own 128 activation rows and half of the BN
//    weight rows, and the pair's MMA reads both halves.
//  * The activation operand is widened by the CTA's widen warps straight
//    into tensor memory (tcgen05.st): one thread owns one activation row, so
//    shared memory carries only the packed activation tile once.
//  * The weight operand is widened in shared memory into the canonical
//    128-byte-swizzled K-major layout, as in the one-SM kernel.
//
// Widening writes each nibble in the high half of a byte (the byte is 16*q)
// and the 32 codes of a 16-byte packed chunk as (even elements, odd
// elements); both operands use that K order, so acc = 256 * sum qa*qw.
//
// Tensor memory per CTA: two BN-column int32 accumulators (the epilogue of
// one tile overlaps the MMAs of the next) and up to four 32-column
// activation stages: 2*BN + 32*stages <= 512.
//
// Warp roles, per CTA (448 threads):
//   warps 0-3   epilogue  (TMEM lanes = the CTA's 128 rows of the tile)
//   warps 4-11  widen     (two groups of four warps taking alternate K
//                          steps: one activation row per thread -> TMEM,
//                          weight chunks -> smem)
//   warp  12    producer  (TMA of the packed tiles; no multicast)
//   warp  13    TMEM allocation; in the even CTA one thread issues the MMAs,
//               in the odd CTA one thread relays "stage widened" to the even
//               CTA (one cluster-scope arrive per stage instead of one per
//               widen warp)
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

constexpr int kStep = 64;          // packed bytes per row per K step (128 codes)
constexpr int kNP = 8;             // packed ring depth
constexpr int kWidenWarps = 8;                 // two groups of four
constexpr int kGroupThreads = 128;
constexpr int kProducerWarp = 4 + kWidenWarps;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kThreads = 32 * (kMmaWarp + 1);

// Widened stages: as many 32-column activation stages as tensor memory holds
// next to two BN-column accumulators, at most 4.
template <int BN>
constexpr int widened_stages() {
  return (512 - 2 * BN) / 32 < 4 ? (512 - 2 * BN) / 32 : 4;
}

struct PairParams {
  const float* scale_a;            // [M]
  const float* scale_b;            // [N]
  __half* Y;
  int64_t ldy;
  int32_t* acc_debug;              // [M x N] or null
  int32_t M, N;
  int32_t kt;                      // K steps
  int32_t tiles_a, tiles_b;        // 256-row tiles, BN-column tiles
  int32_t y_vec_ok;
  int32_t* status;
};

template <int BN>
struct PairSmem {
  static constexpr int kNW = widened_stages<BN>();
  static constexpr int kHalf = BN / 2;                     // weight rows per CTA
  static constexpr int kPackA = 128 * kStep;               // 8 KB, 64-byte swizzle
  static constexpr int kPackB = kHalf * kStep;
  static constexpr int kWideB = kHalf * 2 * kStep;         // SW128 K-major
  static constexpr int off_wide_b = 0;                     // 1024-aligned
  static constexpr int off_pack_a = off_wide_b + kNW * kWideB;
  static constexpr int off_pack_b = off_pack_a + kNP * kPackA;
  static constexpr int off_bar = off_pack_b + kNP * kPackB;
  static constexpr int kNumBars = 2 * kNP + 2 * kNW + 2 + 2 + 1;
  static constexpr int off_misc = off_bar + 8 * kNumBars;
  static constexpr int kBytes = off_misc + 16 + 1024;
};

template <int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                      const __grid_constant__ CUtensorMap map_b, const PairParams p) {
  using S = PairSmem<BN>;
  constexpr int kNW = S::kNW;
  static_assert(BN % 32 == 0 && BN >= 64 && kNW >= 2, "tile width");
  constexpr uint32_t kAcol = 2 * BN;                       // activation stages in TMEM
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::off_bar);
  uint64_t* full_p = bars;                   // local: TMA landed
  uint64_t* empty_p = full_p + kNP;          // local: widen done reading
  uint64_t* full_w = empty_p + kNP;          // widened: 4 local warps (+ the odd CTA's relay)
  uint64_t* empty_w = full_w + kNW;          // each CTA: the pair's MMAs done with the stage
  uint64_t* tmem_full = empty_w + kNW;       // each CTA: accumulator ready
  uint64_t* tmem_empty = tmem_full + 2;      // even CTA: both epilogues drained (8 warps)
  uint64_t* drain = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::off_misc);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + S::off_misc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNP; ++i) { mbar_init(&full_p[i], 1); mbar_init(&empty_p[i], 4); }
    for (int i = 0; i < kNW; ++i) {
      mbar_init(&full_w[i], leader ? 5 : 4);
      mbar_init(&empty_w[i], 1);
    }
    for (int i = 0; i < 2; ++i) { mbar_init(&tmem_full[i], 1); mbar_init(&tmem_empty[i], 8); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0 && p.kt > 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                            // barriers of both CTAs initialized
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = p.tiles_a * p.tiles_b;
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
        const int ta = tile % p.tiles_a, tb = tile / p.tiles_a;
        const int ya = ta * 256 + static_cast<int>(rank) * 128;
        const int yb = tb * BN + static_cast<int>(rank) * S::kHalf;
        for (int ks = 0; ks < p.kt; ++ks, ++it) {
          const uint32_t s = it % kNP, ph = (it / kNP) & 1;
          if (!(ok = mbar_wait_bounded(&empty_p[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
          mbar_arrive_expect_tx(&full_p[s], S::kPackA + S::kPackB);
          tma_load_2d(smem + S::off_pack_a + s * S::kPackA, &map_a, &full_p[s], ks * kStep, ya);
          tma_load_2d(smem + S::off_pack_b + s * S::kPackB, &map_b, &full_p[s], ks * kStep, yb);
        }
      }
      if (!ok)
        for (uint32_t i = (it > kNP ? it - kNP : 0); i < it; ++i)
          mbar_wait_bounded(&full_p[i % kNP], (i / kNP) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA (even CTA)
    if (!leader && lane == 0) {
      // relay: this CTA's stage is widened -> the even CTA's full_w
      const uint32_t full_w0 = mapa_shared(smem_u32(&full_w[0]), 0);
      uint32_t wi = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl)
        for (int ks = 0; ks < p.kt; ++ks, ++wi) {
          const uint32_t s = wi % kNW, ph = (wi / kNW) & 1;
          if (!(ok = mbar_wait_bounded(&full_w[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          // The widen warps fenced their shared-memory and tensor-memory
          // writes and released them on this CTA's barrier, which the wait
          // above acquired; a release at cluster scope here would also wait
          // for the epilogue's outstanding global stores (~0.7 us per stage).
          mbar_arrive_cluster_relaxed(full_w0 + s * 8);
        }
    }
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_i8_m256(BN);
      uint32_t wi = 0, tcount = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++tcount) {
        const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
        if (!(ok = mbar_wait_cluster_bounded(&tmem_empty[buf], tph ^ 1, abort_flag, p.status, kDevTimeoutMma))) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int ks = 0; ks < p.kt; ++ks, ++wi) {
          const uint32_t s = wi % kNW, ph = (wi / kNW) & 1;
          if (!(ok = mbar_wait_cluster_bounded(&full_w[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          tc_fence_after();
          const uint32_t a = tmem_base + kAcol + s * 32;
          const uint64_t db = smem_desc_kmajor(smem_u32(smem + S::off_wide_b + s * S::kWideB), 128);
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_i8_pair_ts(d, a + 8 * k, db + 2 * k, idesc, (ks | k) != 0);
          mma_commit_pair(&empty_w[s], 0x3);
        }
        if (ok) mma_commit_pair(&tmem_full[buf], 0x3);
      }
      mma_commit_pair_local(drain);
      mbar_wait_bounded(drain, 0, abort_flag, p.status, kDevTimeoutDrain, kDrainLimitNs);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ widen
    const int wt = threadIdx.x - 128;
    const int group = wt >> 7;                     // takes K steps with it % 2 == group
    const int arow = wt & 127;                     // = TMEM lane (warp % 4 quadrant)
    const int gt = arow;                           // thread index within the group
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
      for (int ks = 0; ks < p.kt; ++ks, ++it) {
        if ((it & 1) != static_cast<uint32_t>(group)) continue;
        const uint32_t s = it % kNP, ph = (it / kNP) & 1;
        const uint32_t sw = it % kNW, phw = (it / kNW) & 1;
        if (!(ok = mbar_wait_bounded(&full_p[s], ph, abort_flag, p.status, kDevTimeoutWiden))) break;
        if (!(ok = mbar_wait_cluster_bounded(&empty_w[sw], phw ^ 1, abort_flag, p.status, kDevTimeoutWiden))) break;
        // activation row: 64 packed bytes (64-byte swizzled rows) -> 128 s8 in TMEM
        {
          const uint8_t* pa = smem + S::off_pack_a + s * S::kPackA + arow * kStep;
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(pa + ((c ^ ((arow >> 1) & 3)) << 4));
            r[8 * c + 0] = (u.x << 4) & 0xF0F0F0F0u;
            r[8 * c + 1] = (u.y << 4) & 0xF0F0F0F0u;
            r[8 * c + 2] = (u.z << 4) & 0xF0F0F0F0u;
            r[8 * c + 3] = (u.w << 4) & 0xF0F0F0F0u;
            r[8 * c + 4] = u.x & 0xF0F0F0F0u;
            r[8 * c + 5] = u.y & 0xF0F0F0F0u;
            r[8 * c + 6] = u.z & 0xF0F0F0F0u;
            r[8 * c + 7] = u.w & 0xF0F0F0F0u;
          }
          tmem_st_32x32b_x32(tmem_base + lane_off + kAcol + sw * 32, r);
        }
        // weight rows: 16-byte packed chunks -> two 16-byte s8 chunks, SW128
        {
          const uint8_t* pb = smem + S::off_pack_b + s * S::kPackB;
          uint8_t* wb = smem + S::off_wide_b + sw * S::kWideB;
          constexpr int kTasks = S::kHalf * 4;
#pragma unroll 2
          for (int task = gt; task < kTasks; task += kGroupThreads) {
            const int row = task >> 2, c = task & 3;
            const uint4 u = *reinterpret_cast<const uint4*>(pb + row * kStep + c * 16);
            uint4 ev, od;
            ev.x = (u.x << 4) & 0xF0F0F0F0u; od.x = u.x & 0xF0F0F0F0u;
            ev.y = (u.y << 4) & 0xF0F0F0F0u; od.y = u.y & 0xF0F0F0F0u;
            ev.z = (u.z << 4) & 0xF0F0F0F0u; od.z = u.z & 0xF0F0F0F0u;
            ev.w = (u.w << 4) & 0xF0F0F0F0u; od.w = u.w & 0xF0F0F0F0u;
            uint8_t* base = wb + (row >> 3) * 1024 + (row & 7) * 128;
            *reinterpret_cast<uint4*>(base + (((2 * c) ^ (row & 7)) << 4)) = ev;
            *reinterpret_cast<uint4*>(base + (((2 * c + 1) ^ (row & 7)) << 4)) = od;
          }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full_w[sw]);
          mbar_arrive(&empty_p[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int lrow = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tmem_empty0 = mapa_shared(smem_u32(&tmem_empty[0]), 0);
    uint32_t tcount = 0;
    bool ok = true;
    for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++tcount) {
      const int ta = tile % p.tiles_a, tb = tile / p.tiles_a;
      const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
      if (!(ok = mbar_wait_cluster_bounded(&tmem_full[buf], tph, abort_flag, p.status, kDevTimeoutEpilogue))) break;
      tc_fence_after();
      const int m = ta * 256 + static_cast<int>(rank) * 128 + lrow;
      const bool m_ok = m < p.M;
      const float s_row = m_ok ? __ldg(p.scale_a + m) * (1.0f / 256.0f) : 0.0f;
      const uint32_t t_acc = tmem_base + lane_off + buf * BN;
      __half* yrow = p.Y + static_cast<int64_t>(m) * p.ldy;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t acc[32];
        tmem_ld_32x32b_x32(t_acc + c * 32, acc);
        tmem_ld_wait();
        if (p.kt == 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[j] = 0;
        }
        const int n0 = tb * BN + c * 32;
        if (!m_ok) continue;
        uint32_t hp[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float s0 = (n0 + j < p.N) ? __ldg(p.scale_b + n0 + j) : 0.0f;
          const float s1 = (n0 + j + 1 < p.N) ? __ldg(p.scale_b + n0 + j + 1) : 0.0f;
          const __half2 h2 = __floats2half2_rn(
              static_cast<float>(static_cast<int32_t>(acc[j])) * s_row * s0,
              static_cast<float>(static_cast<int32_t>(acc[j + 1])) * s_row * s1);
          hp[j / 2] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        if (p.y_vec_ok && n0 + 32 <= p.N) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(yrow + n0 + 8 * q) =
                make_uint4(hp[4 * q], hp[4 * q + 1], hp[4 * q + 2], hp[4 * q + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (n0 + j < p.N)
              reinterpret_cast<uint16_t*>(yrow)[n0 + j] = static_cast<uint16_t>(hp[j / 2] >> (16 * (j & 1)));
        }
        if (p.acc_debug != nullptr) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (n0 + j < p.N)
              p.acc_debug[static_cast<int64_t>(m) * p.N + n0 + j] = static_cast<int32_t>(acc[j]) >> 8;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty0 + buf * 8);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                            // no CTA leaves while its pair may still signal it
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <int BN>
cudaError_t run_pair(const CUtensorMap& ma, const CUtensorMap& mb, const PairParams& p,
                     cudaStream_t stream) {
  auto k = w4a4_gemm_pair_kernel<BN>;
  const int smem = PairSmem<BN>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int clusters = std::min(p.tiles_a * p.tiles_b, sm_count() / 2);
  k<<<2 * clusters, kThreads, smem, stream>>>(ma, mb, p);
  return cudaGetLastError();
}

}  // namespace

// Tile width for the pair kernel: the fewest tile rounds over the SM pairs,
// weighted by the width (one round of a BN-wide tile costs about BN).
int pair_tile_width(int64_t M, int64_t N, int sms) {
  const int64_t ta = (M + 255) / 256;
  const int cands[] = {192, 160, 128};
  int64_t cost[3];
  int64_t best_cost = -1;
  for (int i = 0; i < 3; ++i) {
    const int bn = cands[i];
    const int64_t tiles = ta * ((N + bn - 1) / bn);
    const int64_t rounds = (tiles + sms / 2 - 1) / (sms / 2);
    cost[i] = rounds * bn;
    if (best_cost < 0 || cost[i] < best_cost) best_cost = cost[i];
  }
  // the widest tile within 2% of the cheapest (wider tiles reuse operands more)
  for (int i = 0; i < 3; ++i)
    if (cost[i] * 100 <= best_cost * 102) return cands[i];
  return 128;
}

qr_status launch_w4a4_gemm_pair(const GemmJob& j, cudaStream_t stream) {
  const int bn = pair_tile_width(j.M, j.N, sm_count());
  PairParams p{};
  p.scale_a = j.a_scales;
  p.scale_b = j.w_scales;
  p.Y = reinterpret_cast<__half*>(j.Y);
  p.ldy = j.ldy;
  p.acc_debug = j.acc_debug;
  p.M = static_cast<int32_t>(j.M);
  p.N = static_cast<int32_t>(j.N);
  p.kt = static_cast<int32_t>(j.Kp / 128);
  p.tiles_a = static_cast<int32_t>((j.M + 255) / 256);
  p.tiles_b = static_cast<int32_t>((j.N + bn - 1) / bn);
  p.y_vec_ok = (reinterpret_cast<uintptr_t>(j.Y) % 16 == 0) && (j.ldy % 8 == 0);
  p.status = device_status_word();
  if (p.status == nullptr) return QR_ERR_CUDA;
  CUtensorMap ma{}, mb{};
  const uint64_t kb = static_cast<uint64_t>(j.Kp) / 2;
  if (p.kt > 0 &&
      (!make_tensor_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.a_codes, kb, j.M, kb, kStep, 128,
                           CU_TENSOR_MAP_SWIZZLE_64B) ||
       !make_tensor_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.w_codes, kb, j.N, kb, kStep,
                           bn / 2, CU_TENSOR_MAP_SWIZZLE_NONE)))
    return QR_ERR_CUDA;
  cudaError_t e;
  switch (bn) {
    case 192: e = run_pair<192>(ma, mb, p, stream); break;
    case 160: e = run_pair<160>(ma, mb, p, stream); break;
    default: e = run_pair<128>(ma, mb, p, stream); break;
  }
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
