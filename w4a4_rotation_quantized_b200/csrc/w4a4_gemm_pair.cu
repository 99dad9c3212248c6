// w4a4_gemm_pair.cu -- the W4A4 linear on pairs of SMs.
//
// Same computation as w4a4_gemm.cu (QUIK §1 and §4: INT4 codes multiplied on
// integer tensor cores with INT32 accumulation, dequantized per token and per
// channel in the epilogue, plus the fp16 product of the outlier columns),
// arranged to move fewer bytes through shared memory per MMA:
//
//  * tcgen05.mma.cta_group::2: the two CTAs of a cluster compute a 256 x BN
//    tile; each CTA holds its own 128 rows of the "A" operand and half of the
//    BN rows of the "B" operand, and the pair's MMA reads both halves.
//  * The A operand is widened by the CTA's widen warps straight into tensor
//    memory (tcgen05.st): one thread owns one row, so shared memory carries
//    only the packed A tile once.
//  * The B operand is widened in shared memory into the canonical
//    128-byte-swizzled K-major layout.
//  * A = activations (M > 64), B = weights.
//  * The packed tiles arrive by TMA in 128-byte rows: a ring slot, and a
//    widened stage, holds two K steps (256 codes), so the MMA thread waits,
//    fences and commits once per eight MMAs.
//  * OUT: the fp16 outlier columns run as a second cta_group::2 MMA of
//    kind::f16 into an fp32 accumulator in TMEM, added in the epilogue.
//
// Widening writes each nibble in the high half of a byte (the byte is 16*q)
// and the 32 codes of a 16-byte packed chunk as (even elements, odd
// elements); both operands use that K order, so acc = 256 * sum qa*qw.
//
// Tensor memory per CTA: two accumulator buffers (the epilogue of one tile
// overlaps the MMAs of the next) of BN int32 columns, plus BN fp32 outlier
// columns when OUT, and up to four 64-column A stages.
//
// Warp roles, per CTA (448 threads):
//   warps 0-3   epilogue  (TMEM lanes = the CTA's 128 A rows of the tile)
//   warps 4-11  widen     (two groups of four warps taking alternate ring
//                          slots: one A row per thread -> TMEM, B chunks ->
//                          smem)
//   warp  12    producer  (TMA of the packed and outlier tiles; no multicast)
//   warp  13    TMEM allocation; in the even CTA one thread issues the MMAs,
//               in the odd CTA one thread relays "stage ready" to the even
//               CTA (one relaxed cluster-scope arrive per stage)
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

constexpr int kStep = 64;          // packed bytes per row per K step (128 codes)
constexpr int kSlot = 2 * kStep;   // packed bytes per row per ring slot (two K steps)
constexpr int kNP = 4;             // packed ring depth (slots)
constexpr int kNO = 2;             // outlier ring depth
constexpr int kOutCols = 32;       // fp16 outlier columns per step (64-byte rows)
constexpr int kWidenWarps = 8;     // two groups of four
constexpr int kGroupThreads = 128;
constexpr int kProducerWarp = 4 + kWidenWarps;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kThreads = 32 * (kMmaWarp + 1);

// A stages: as many 64-column stages (two K steps) as tensor memory holds
// next to the two accumulator buffers, at most 4.
template <int BN, bool OUT>
constexpr int widened_stages() {
  return (512 - (OUT ? 4 : 2) * BN) / 64 < 4 ? (512 - (OUT ? 4 : 2) * BN) / 64 : 4;
}

struct PairParams {
  const float* scale_a;            // per A-side row
  const float* scale_b;            // per B-side row
  const int32_t* a_zeros;          // asymmetric activations: zero point per row, else null
  const int32_t* w_sums;           // with a_zeros: code sum per weight row
  __half* Y;
  int64_t ldy;
  int32_t* acc_debug;              // [M x N] or null
  int32_t rows_a, rows_b;          // A-side and B-side row counts
  int32_t M, N;                    // output shape
  int32_t kt, ot;                  // int4 K steps, outlier steps
  int32_t tiles_a, tiles_b;        // 256-row A tiles, BN-row B tiles
  int32_t y_vec_ok;
  int32_t y_tma;                   // Y leaves through tensor stores (map_y is valid)
  int32_t* status;
};

template <int BN, bool OUT>
struct PairSmem {
  static constexpr int kNW = widened_stages<BN, OUT>();
  static constexpr int kHalf = BN / 2;                     // B rows per CTA
  static constexpr int kPackA = 128 * kSlot;               // 16 KB, 128-byte swizzle
  static constexpr int kPackB = kHalf * kSlot;             // 128-byte swizzle
  static constexpr int kWideBlk = kHalf * 128;             // one SW128 K-major block (128 codes)
  static constexpr int kWideB = 2 * kWideBlk;              // a stage: two K blocks
  static constexpr int kOutA = OUT ? 128 * kOutCols * 2 : 0;     // SW64 K-major
  static constexpr int kOutB = OUT ? kHalf * kOutCols * 2 : 0;
  static constexpr int off_wide_b = 0;                     // 1024-aligned
  static constexpr int off_out_a = off_wide_b + kNW * kWideB;
  static constexpr int off_out_b = off_out_a + kNO * kOutA;
  static constexpr int off_pack_a = off_out_b + kNO * kOutB;
  static constexpr int off_pack_b = off_pack_a + kNP * kPackA;
  // epilogue: per warp, two staging boxes of 32 rows x 32 fp16 columns
  // (64-byte swizzle, for the tensor store) and the tile's B-side scales
  // (and, asymmetric, code sums) as floats
  static constexpr int kYBox = 32 * 64;
  static constexpr int kSbFloats = 2 * BN;
  static constexpr int off_ystage = off_pack_b + kNP * kPackB;
  static constexpr int off_sb = off_ystage + 4 * 2 * kYBox;
  static constexpr int off_bar = off_sb + 4 * kSbFloats * 4;
  // full_p, empty_p, full_w, empty_w, full_o, full_o2, empty_o,
  // tmem_full[2], tmem_empty[2], drain
  static constexpr int kNumBars = 2 * kNP + 2 * kNW + 3 * kNO + 5;
  static constexpr int off_misc = off_bar + 8 * kNumBars;
  static constexpr int kBytes = off_misc + 16 + 1024;
  static_assert(off_out_a % 1024 == 0 && off_out_b % 1024 == 0 && off_pack_a % 1024 == 0 &&
                    kPackB % 1024 == 0 && off_ystage % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

template <int BN, bool OUT, bool ASYM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                      const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_oa,
                      const __grid_constant__ CUtensorMap map_ob,
                      const __grid_constant__ CUtensorMap map_y, const PairParams p) {
  using S = PairSmem<BN, OUT>;
  constexpr int kNW = S::kNW;
  static_assert(BN % 32 == 0 && BN >= 32 && kNW >= 2 && S::kWideBlk % 1024 == 0, "tile width");
  constexpr uint32_t kColsAcc = OUT ? 2 * BN : BN;         // per accumulator buffer
  constexpr uint32_t kAcol = 2 * kColsAcc;                 // A stages in TMEM
  static_assert(kAcol + 64 * kNW <= 512, "tensor memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::off_bar);
  uint64_t* full_p = bars;                   // local: TMA landed
  uint64_t* empty_p = full_p + kNP;          // local: the widen group done reading
  uint64_t* full_w = empty_p + kNP;          // widened: 4 local warps (+ the odd CTA's relay)
  uint64_t* empty_w = full_w + kNW;          // each CTA: the pair's MMAs done with the stage
  uint64_t* full_o = empty_w + kNW;          // local: outlier TMA landed
  uint64_t* full_o2 = full_o + kNO;          // even CTA: the odd CTA's outlier TMA landed
  uint64_t* empty_o = full_o2 + kNO;         // each CTA: the pair's MMAs done with the stage
  uint64_t* tmem_full = empty_o + kNO;       // each CTA: accumulator ready
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
    for (int i = 0; i < kNO; ++i) {
      mbar_init(&full_o[i], 1);
      mbar_init(&full_o2[i], 1);
      mbar_init(&empty_o[i], 1);
    }
    for (int i = 0; i < 2; ++i) { mbar_init(&tmem_full[i], 1); mbar_init(&tmem_empty[i], 8); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    if (p.kt > 0) { tma_prefetch_desc(&map_a); tma_prefetch_desc(&map_b); }
    if (OUT && p.ot > 0) { tma_prefetch_desc(&map_oa); tma_prefetch_desc(&map_ob); }
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
  grid_dep_wait();                           // the previous kernel's outputs are visible
  grid_dep_launch();

  const int num_tiles = p.tiles_a * p.tiles_b;
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const int slots = (p.kt + 1) >> 1;         // ring slots per tile

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0, ot = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
        const int ta = tile % p.tiles_a, tb = tile / p.tiles_a;
        const int ya = ta * 256 + static_cast<int>(rank) * 128;
        const int yb = tb * BN + static_cast<int>(rank) * S::kHalf;
        for (int ps = 0; ps < slots; ++ps, ++it) {
          const uint32_t s = it % kNP, ph = (it / kNP) & 1;
          if (!(ok = mbar_wait_bounded(&empty_p[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
          mbar_arrive_expect_tx(&full_p[s], S::kPackA + S::kPackB);
          tma_load_2d(smem + S::off_pack_a + s * S::kPackA, &map_a, &full_p[s], ps * kSlot, ya);
          tma_load_2d(smem + S::off_pack_b + s * S::kPackB, &map_b, &full_p[s], ps * kSlot, yb);
        }
        if (OUT)
          for (int os = 0; os < p.ot && ok; ++os, ++ot) {
            const uint32_t s = ot % kNO, ph = (ot / kNO) & 1;
            if (!(ok = mbar_wait_cluster_bounded(&empty_o[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
            mbar_arrive_expect_tx(&full_o[s], S::kOutA + S::kOutB);
            tma_load_2d(smem + S::off_out_a + s * S::kOutA, &map_oa, &full_o[s], os * kOutCols, ya);
            tma_load_2d(smem + S::off_out_b + s * S::kOutB, &map_ob, &full_o[s], os * kOutCols, yb);
          }
      }
      if (!ok) {
        for (uint32_t i = (it > kNP ? it - kNP : 0); i < it; ++i)
          mbar_wait_bounded(&full_p[i % kNP], (i / kNP) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
        for (uint32_t i = (ot > kNO ? ot - kNO : 0); i < ot; ++i)
          mbar_wait_bounded(&full_o[i % kNO], (i / kNO) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    if (!leader && lane == 0) {
      // ------------------------------------------------------------ relay (odd CTA)
      // This CTA's stages are ready -> the even CTA's barriers.  The local
      // waits acquire the widen warps' fenced writes and the TMA's
      // completion; a release at cluster scope here would also wait for the
      // epilogue's outstanding global stores (~0.7 us per stage).
      const uint32_t full_w0 = mapa_shared(smem_u32(&full_w[0]), 0);
      const uint32_t full_o20 = mapa_shared(smem_u32(&full_o2[0]), 0);
      uint32_t wi = 0, oi = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
        for (int ps = 0; ps < slots; ++ps, ++wi) {
          const uint32_t s = wi % kNW, ph = (wi / kNW) & 1;
          if (!(ok = mbar_wait_bounded(&full_w[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          mbar_arrive_cluster_relaxed(full_w0 + s * 8);
        }
        if (OUT)
          for (int os = 0; os < p.ot && ok; ++os, ++oi) {
            const uint32_t s = oi % kNO, ph = (oi / kNO) & 1;
            if (!(ok = mbar_wait_bounded(&full_o[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
            mbar_arrive_cluster_relaxed(full_o20 + s * 8);
          }
      }
    }
    if (leader && lane == 0) {
      // ------------------------------------------------------------ MMA (even CTA)
      constexpr uint32_t idesc = idesc_i8_m256(BN);
      constexpr uint32_t idesc_o = idesc_f16_m256(BN);
      uint32_t wi = 0, oi = 0, tcount = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++tcount) {
        const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
        if (!(ok = mbar_wait_cluster_bounded(&tmem_empty[buf], tph ^ 1, abort_flag, p.status, kDevTimeoutMma))) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * kColsAcc;
        for (int ps = 0; ps < slots; ++ps, ++wi) {
          const uint32_t s = wi % kNW, ph = (wi / kNW) & 1;
          if (!(ok = mbar_wait_cluster_bounded(&full_w[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
          tc_fence_after();
          // two K steps; past K (odd step count) both operands are zero-filled
          const uint32_t a = tmem_base + kAcol + s * 64;
          const uint64_t db0 = smem_desc_kmajor(smem_u32(smem + S::off_wide_b + s * S::kWideB), 128);
          const uint64_t db1 = smem_desc_kmajor(smem_u32(smem + S::off_wide_b + s * S::kWideB + S::kWideBlk), 128);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_i8_pair_ts(d, a + 8 * k, (k < 4 ? db0 : db1) + 2 * (k & 3), idesc, (ps | k) != 0);
          mma_commit_pair(&empty_w[s], 0x3);
        }
        if (OUT && ok)
          for (int os = 0; os < p.ot; ++os, ++oi) {
            const uint32_t s = oi % kNO, ph = (oi / kNO) & 1;
            if (!(ok = mbar_wait_cluster_bounded(&full_o[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
            if (!(ok = mbar_wait_cluster_bounded(&full_o2[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
            tc_fence_after();
            const uint64_t da = smem_desc_kmajor(smem_u32(smem + S::off_out_a + s * S::kOutA), 64);
            const uint64_t db = smem_desc_kmajor(smem_u32(smem + S::off_out_b + s * S::kOutB), 64);
#pragma unroll
            for (int k = 0; k < 2; ++k) mma_f16_pair(d + BN, da + 2 * k, db + 2 * k, idesc_o, (os | k) != 0);
            mma_commit_pair(&empty_o[s], 0x3);
          }
        if (ok) mma_commit_pair(&tmem_full[buf], 0x3);
      }
      mma_commit_pair_local(drain);
      mbar_wait_bounded(drain, 0, abort_flag, p.status, kDevTimeoutDrain, kDrainLimitNs);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ widen
    const int wt = threadIdx.x - 128;
    const int group = wt >> 7;                     // takes the ring slots wi with wi % 2 == group
    const int arow = wt & 127;                     // = TMEM lane (warp % 4 quadrant)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t pi = 0;                               // slots (= stages) of the earlier tiles
    bool ok = true;
    for (int tile = cid; tile < num_tiles && ok; tile += ncl, pi += slots) {
      // Parity of the global slot index, not of the slot within the tile:
      // a group must never run two uses of a stage ahead of the MMAs, or
      // the parity wait on empty_w would pass a phase early (with two
      // stages and an odd slot count, per-tile parity lets it).
      for (int ps = (group + static_cast<int>(pi)) & 1; ps < slots; ps += 2) {
        const uint32_t wi = pi + ps;
        const uint32_t s = wi % kNP, ph = (wi / kNP) & 1;
        const uint32_t sw = wi % kNW, phw = (wi / kNW) & 1;
        if (!(ok = mbar_wait_bounded(&full_p[s], ph, abort_flag, p.status, kDevTimeoutWiden))) break;
        if (!(ok = mbar_wait_cluster_bounded(&empty_w[sw], phw ^ 1, abort_flag, p.status, kDevTimeoutWiden))) break;
        // A row: 128 packed bytes (128-byte swizzled rows) -> 256 s8 in TMEM
        {
          const uint8_t* pa = smem + S::off_pack_a + s * S::kPackA + arow * kSlot;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 u = *reinterpret_cast<const uint4*>(pa + (((4 * h + c) ^ (arow & 7)) << 4));
              r[8 * c + 0] = (u.x << 4) & 0xF0F0F0F0u;
              r[8 * c + 1] = (u.y << 4) & 0xF0F0F0F0u;
              r[8 * c + 2] = (u.z << 4) & 0xF0F0F0F0u;
              r[8 * c + 3] = (u.w << 4) & 0xF0F0F0F0u;
              r[8 * c + 4] = u.x & 0xF0F0F0F0u;
              r[8 * c + 5] = u.y & 0xF0F0F0F0u;
              r[8 * c + 6] = u.z & 0xF0F0F0F0u;
              r[8 * c + 7] = u.w & 0xF0F0F0F0u;
            }
            tmem_st_32x32b_x32(tmem_base + lane_off + kAcol + sw * 64 + 32 * h, r);
          }
        }
        // B rows (128-byte swizzled): each 16-byte packed chunk -> two 16-byte
        // s8 chunks of the K block it belongs to, SW128
        {
          const uint8_t* pb = smem + S::off_pack_b + s * S::kPackB;
          uint8_t* wb = smem + S::off_wide_b + sw * S::kWideB;
          constexpr int kTasks = S::kHalf * 4;
#pragma unroll 1
          for (int task = arow; task < kTasks; task += kGroupThreads) {
            // eight consecutive threads take eight consecutive rows (one
            // 128-byte swizzle atom) at the same chunk c: their 16-byte reads
            // (chunk (4h + c) ^ row) and writes ((2c, 2c+1) ^ row) then fall in
            // eight distinct bank groups
            const int row = (task & 7) | ((task >> 5) << 3), c = (task >> 3) & 3;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 u = *reinterpret_cast<const uint4*>(pb + row * kSlot + (((4 * h + c) ^ (row & 7)) << 4));
              uint4 ev, od;
              ev.x = (u.x << 4) & 0xF0F0F0F0u; od.x = u.x & 0xF0F0F0F0u;
              ev.y = (u.y << 4) & 0xF0F0F0F0u; od.y = u.y & 0xF0F0F0F0u;
              ev.z = (u.z << 4) & 0xF0F0F0F0u; od.z = u.z & 0xF0F0F0F0u;
              ev.w = (u.w << 4) & 0xF0F0F0F0u; od.w = u.w & 0xF0F0F0F0u;
              uint8_t* base = wb + h * S::kWideBlk + (row >> 3) * 1024 + (row & 7) * 128;
              *reinterpret_cast<uint4*>(base + (((2 * c) ^ (row & 7)) << 4)) = ev;
              *reinterpret_cast<uint4*>(base + (((2 * c + 1) ^ (row & 7)) << 4)) = od;
            }
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
    // Lane = A-side row (output row m), 32 output columns per chunk.  The
    // tile's B-side scales sit in a per-warp shared-memory copy (read as
    // broadcast float4); the fp16 results go to a per-warp 32 x 32 staging
    // box that one lane hands to a tensor store, double-buffered, so the
    // warp never issues scattered global stores.
    const int lrow = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tmem_empty0 = mapa_shared(smem_u32(&tmem_empty[0]), 0);
    float* sb_w = reinterpret_cast<float*>(smem + S::off_sb) + warp * S::kSbFloats;
    uint8_t* ystage = smem + S::off_ystage + warp * 2 * S::kYBox;
    uint32_t tcount = 0, nbox = 0;
    bool ok = true;
    for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++tcount) {
      const int ta = tile % p.tiles_a, tb = tile / p.tiles_a;
      const uint32_t buf = tcount & 1, tph = (tcount >> 1) & 1;
      __syncwarp();                                // the previous tile's readers are done
      for (int i = lane; i < BN; i += 32) {
        const int n = tb * BN + i;
        const bool n_ok = n < p.rows_b;
        sb_w[i] = n_ok ? __ldg(p.scale_b + n) : 0.0f;
        if (ASYM) sb_w[BN + i] = n_ok ? static_cast<float>(__ldg(p.w_sums + n)) : 0.0f;
      }
      __syncwarp();
      if (!(ok = mbar_wait_cluster_bounded(&tmem_full[buf], tph, abort_flag, p.status, kDevTimeoutEpilogue))) break;
      tc_fence_after();
      const int ra = ta * 256 + static_cast<int>(rank) * 128 + lrow;   // A-side row
      const bool ra_ok = ra < p.rows_a;
      const float s_row = ra_ok ? __ldg(p.scale_a + ra) * (1.0f / 256.0f) : 0.0f;
      // asymmetric activations: acc - 256 * zero * w_sum (the accumulator is 256 x)
      const float zrow = (ASYM && ra_ok) ? 256.0f * static_cast<float>(__ldg(p.a_zeros + ra)) : 0.0f;
      const uint32_t t_acc = tmem_base + lane_off + buf * kColsAcc;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t acc[32];
        uint32_t oacc[32];
        tmem_ld_32x32b_x32(t_acc + c * 32, acc);
        if (OUT) tmem_ld_32x32b_x32(t_acc + BN + c * 32, oacc);
        tmem_ld_wait();
        const bool kz = p.kt == 0, oz = OUT && p.ot == 0;
        const int cb0 = tb * BN + c * 32;          // first B-side row (output column) of the chunk
        const float4* sb4 = reinterpret_cast<const float4*>(sb_w + c * 32);
        const float4* ws4 = reinterpret_cast<const float4*>(sb_w + BN + c * 32);
        uint32_t hp[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 sb = sb4[q];
          const float sbv[4] = {sb.x, sb.y, sb.z, sb.w};
          float wsv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          if (ASYM) {
            const float4 w = ws4[q];
            wsv[0] = w.x; wsv[1] = w.y; wsv[2] = w.z; wsv[3] = w.w;
          }
          float y[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int j = 4 * q + t;
            float a = kz ? 0.0f : static_cast<float>(static_cast<int32_t>(acc[j]));
            if (ASYM) a = fmaf(-zrow, wsv[t], a);
            y[t] = a * s_row * sbv[t];
            if (OUT && !oz) y[t] += __uint_as_float(oacc[j]);
          }
          const __half2 h0 = __floats2half2_rn(y[0], y[1]);
          const __half2 h1 = __floats2half2_rn(y[2], y[3]);
          hp[2 * q] = *reinterpret_cast<const uint32_t*>(&h0);
          hp[2 * q + 1] = *reinterpret_cast<const uint32_t*>(&h1);
        }
        if (p.y_tma) {
          // box row = lane: 64 bytes as four 16-byte chunks, chunk index
          // XOR (row / 2) % 4 (the 64-byte swizzle of the tensor map)
          uint8_t* box = ystage + (nbox & 1) * S::kYBox;
          if (lane == 0 && nbox >= 2) bulk_wait_group_read<1>();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(box + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(hp[4 * q], hp[4 * q + 1], hp[4 * q + 2], hp[4 * q + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&map_y, box, cb0, ta * 256 + static_cast<int>(rank) * 128 + warp * 32);
            bulk_commit_group();
          }
          ++nbox;
        } else if (ra_ok) {
          __half* yrow = p.Y + static_cast<int64_t>(ra) * p.ldy;
          if (p.y_vec_ok && cb0 + 32 <= p.rows_b) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(yrow + cb0 + 8 * q) =
                  make_uint4(hp[4 * q], hp[4 * q + 1], hp[4 * q + 2], hp[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (cb0 + j < p.rows_b)
                reinterpret_cast<uint16_t*>(yrow)[cb0 + j] =
                    static_cast<uint16_t>(hp[j / 2] >> (16 * (j & 1)));
          }
        }
        if (p.acc_debug != nullptr && ra_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cb0 + j < p.rows_b)
              p.acc_debug[static_cast<int64_t>(ra) * p.N + cb0 + j] =
                  kz ? 0 : static_cast<int32_t>(acc[j]) >> 8;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty0 + buf * 8);
    }
    if (lane == 0) bulk_wait_group<0>();           // tensor stores done before the CTA ends
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                            // no CTA leaves while its pair may still signal it
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <int BN, bool OUT>
cudaError_t run_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& moa,
                     const CUtensorMap& mob, const CUtensorMap& my, const PairParams& p,
                     cudaStream_t stream) {
  auto k = p.a_zeros != nullptr ? w4a4_gemm_pair_kernel<BN, OUT, true>
                                : w4a4_gemm_pair_kernel<BN, OUT, false>;
  const int smem = PairSmem<BN, OUT>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int clusters = std::min(p.tiles_a * p.tiles_b, sm_count() / 2);
  e = launch_pdl(k, dim3(2 * clusters), dim3(kThreads), smem, stream, 1, ma, mb, moa, mob, my, p);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace

// Tile width without outlier columns: 160 or 128 (both leave tensor memory
// for at least three A stages next to the double-buffered accumulator; 192
// would leave two, too shallow to hide the widen).  Cost = tile rounds over
// the SM pairs x (width + a per-step overhead worth ~64 columns); the wider
// tile wins within 2%.
int pair_tile_width(int64_t M, int64_t N, int sms) {
  const int64_t ta = (M + 255) / 256;
  const int cands[] = {160, 128};
  int64_t cost[2];
  for (int i = 0; i < 2; ++i) {
    const int64_t tiles = ta * ((N + cands[i] - 1) / cands[i]);
    const int64_t rounds = (tiles + sms / 2 - 1) / (sms / 2);
    cost[i] = rounds * (cands[i] + 64);
  }
  return cost[0] * 100 <= cost[1] * 102 ? 160 : 128;
}

qr_status launch_w4a4_gemm_pair(const GemmJob& j, cudaStream_t stream) {
  const bool out = j.n_out > 0;
  const int bn = out ? 96 : pair_tile_width(j.M, j.N, sm_count());
  PairParams p{};
  p.scale_a = j.a_scales;
  p.scale_b = j.w_scales;
  p.a_zeros = j.a_zeros;
  p.w_sums = j.w_sums;
  p.Y = reinterpret_cast<__half*>(j.Y);
  p.ldy = j.ldy;
  p.acc_debug = j.acc_debug;
  p.rows_a = static_cast<int32_t>(j.M);
  p.rows_b = static_cast<int32_t>(j.N);
  p.M = static_cast<int32_t>(j.M);
  p.N = static_cast<int32_t>(j.N);
  p.kt = static_cast<int32_t>(j.Kp / 128);
  p.ot = out ? (j.n_out + kOutCols - 1) / kOutCols : 0;
  p.tiles_a = static_cast<int32_t>((j.M + 255) / 256);
  p.tiles_b = static_cast<int32_t>((j.N + bn - 1) / bn);
  p.y_vec_ok = (reinterpret_cast<uintptr_t>(j.Y) % 16 == 0) && (j.ldy % 8 == 0);
  // Y through tensor stores: boxes of 32 columns x 32 rows, 64-byte swizzle
  CUtensorMap my{};
  p.y_tma = p.y_vec_ok &&
            make_tensor_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.Y, static_cast<uint64_t>(j.N),
                               static_cast<uint64_t>(j.M), static_cast<uint64_t>(j.ldy) * 2, 32, 32,
                               CU_TENSOR_MAP_SWIZZLE_64B);
  p.status = device_status_word();
  if (p.status == nullptr) return QR_ERR_CUDA;
  CUtensorMap ma{}, mb{}, moa{}, mob{};
  const uint64_t kb = static_cast<uint64_t>(j.Kp) / 2;   // packed bytes per row
  if (p.kt > 0 &&
      (!make_tensor_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.a_codes, kb, j.M, kb, kSlot, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
       !make_tensor_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.w_codes, kb, j.N, kb, kSlot,
                           bn / 2, CU_TENSOR_MAP_SWIZZLE_128B)))
    return QR_ERR_CUDA;
  if (out) {
    const uint64_t no = static_cast<uint64_t>(j.n_out);
    if (!make_tensor_map_2d(&moa, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.x_out, no, j.M, no * 2,
                            kOutCols, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_tensor_map_2d(&mob, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.w_out, no, j.N, no * 2,
                            kOutCols, bn / 2, CU_TENSOR_MAP_SWIZZLE_64B))
      return QR_ERR_CUDA;
  }
  cudaError_t e;
  if (out) {
    e = run_pair<96, true>(ma, mb, moa, mob, my, p, stream);
  } else {
    e = bn == 160 ? run_pair<160, false>(ma, mb, moa, mob, my, p, stream)
                  : run_pair<128, false>(ma, mb, moa, mob, my, p, stream);
  }
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
