// w4a4_gemm_decode.cu -- the W4A4 linear for a few tokens (M <= 64).
//
// Same computation as the prefill kernels (QUIK §1 and §4: INT4 codes
// multiplied on integer tensor cores with INT32 accumulation, dequantized
// per token and per channel, plus the fp16 product of the outlier columns),
// shaped for decode, where the packed weights are nearly all of the bytes:
//
//  * Operands swapped: the MMA's M side is 128 weight rows, widened by the
//    widen warps straight into tensor memory; the tokens (BN = 32 or 64
//    rows, zero-filled beyond M) are the shared-memory B operand.
//  * One 128-row weight tile per cluster and K split over the cluster's KS
//    CTAs (KS = 1, 2 or 4, chosen so that tiles x KS fills the SMs): CTA r
//    runs a contiguous range of the K steps.  The partial sums are then
//    exchanged, not funnelled: CTA r owns the rows [r*128/KS, (r+1)*128/KS)
//    of the tile; every CTA stages the other CTAs' rows of its int32
//    partials in its own shared memory and sends each warp's 32 rows with
//    one shared-to-shared bulk copy into the owner's receive slot, and each
//    CTA adds the partials of its own rows (integer adds: the order does not
//    matter) and runs their epilogue, ending in one tensor store of the fp16
//    [token][row] box.  The fp16 outlier steps all run in CTA 0, which sends
//    the fp32 outlier sums with its partials, so that sum has one order.
//  * One CTA per SM runs a deep ring of widened stages (the chain widen ->
//    MMA -> stage free is local to the SM).
//
// Warp roles (448 threads):
//   warps 0-3   epilogue (TMEM lane = weight row of the tile)
//   warps 4-11  widen (two groups of four warps taking alternate K steps)
//   warp  12    producers (TMA; no multicast): lane 0 the packed ring, lane 1
//               the fp16 outlier ring, whose steps the MMA thread interleaves
//               with the int steps
//   warp  13    TMEM allocation and the MMA-issuing thread
//
// Fused variant (ROT): the kernel first rotates and quantizes the token rows
// itself (warps 0-11, whole rows per CTA, in the wide-B area of shared
// memory before the ring starts), writes their codes, scales and outlier
// columns to global memory, and meets the other CTAs at a grid-wide barrier;
// meanwhile the producer has already put the weight halves of the first ring
// slots in flight.  The token halves of the ring and the token scales are
// read after the barrier.  One launch per decode step instead of two.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>

#include "qr_device.cuh"
#include "qr_internal.h"
#include "row_quant.cuh"

namespace qr {

namespace {

constexpr int kStep = 64;          // packed bytes per row per K step (128 codes)
constexpr int kSlot = 2 * kStep;   // packed bytes per row per ring slot (two K steps)
constexpr int kNP = 4;             // packed ring depth (slots)
constexpr int kNO = 2;             // outlier ring depth
constexpr int kOutCols = 32;       // fp16 outlier columns per step (64-byte rows)
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kThreads = 32 * 14;
constexpr int kSmemBudget = 227 * 1024;

// The token rows of a decode step as the fused kernel takes them: the same
// steps as the row kernels (FlatQuant "模型架构": the online transform and
// the quantization fused into the kernel that consumes them; QUIK "性能分析":
// the separate quantization pass is what keeps the measured speedup below
// the ideal one).  Kept columns of QUIK §1 gathered in order, the optional
// random-sign diagonal, Walsh-Hadamard butterflies per block in fp32 (QuaRot
// §2), the row absmax (or min and max) and its scale, round-half-to-even
// codes packed two per byte, the GSR sequency order by a gather at packing.
struct FusedRows {
  const __half* src;               // tokens [M x ld] fp16
  int64_t ld;
  int32_t K, Kr, Kp, n_out;        // Kr = K - n_out rotated columns, Kp packed width
  const int32_t* outlier_idx;      // ascending [n_out], or null
  const int8_t* signs;             // random-sign diagonal [Kp], or null
  int32_t lb, gsr, aligned;        // log2 block, sequency order, 16-byte rows
  int32_t padded;                  // scatter through the padded buffer (room permitting)
  float clip_ratio, inv_sqrt_block;
  uint8_t* codes;                  // [M x Kp/2]: written here, read back by the ring
  float* scales;                   // [M]
  int32_t* zeros;                  // [M] zero points (asymmetric) or null
  __half* out16;                   // [M x n_out] or null
  uint32_t* sync;                  // grid barrier words [2]
};

struct DecodeParams {
  const float* w_scales;           // [N]
  const float* a_scales;           // [M]
  const int32_t* a_zeros;          // asymmetric activations: zero point per token [M], else null
  const int32_t* w_sums;           // with a_zeros: code sum per weight row [N]
  __half* Y;
  int64_t ldy;
  int32_t* acc_debug;              // [M x N] or null
  int32_t N, M;
  int32_t kt, ot;                  // int4 K steps, outlier steps
  int32_t ks;                      // CTAs splitting K in a cluster
  int32_t y_tma;                   // Y leaves through tensor stores (map_y is valid)
  int32_t* status;
  FusedRows rows;                  // the fused kernel's token rows
};

template <int BN, bool OUT>
struct DecodeLayout {
  static constexpr int kPackA = 128 * kSlot;               // 16 KB, 128-byte swizzle
  static constexpr int kPackB = BN * kSlot;                // 128-byte swizzle
  static constexpr int kWideBlk = BN * 128;                // one SW128 K-major block (128 codes)
  static constexpr int kWideB = 2 * kWideBlk;              // a stage: two K blocks
  static constexpr int kOutA = OUT ? 128 * kOutCols * 2 : 0;     // SW64 K-major
  static constexpr int kOutB = OUT ? BN * kOutCols * 2 : 0;
  // partials received from the other CTAs of the cluster: (KS-1) slots of
  // 128/KS rows, each row BN int32 (+ BN fp32 outlier sums) + 4 words of
  // padding (an odd number of 16-byte chunks per row: conflict-free rows)
  static constexpr int kMaxKS = BN == 64 ? 2 : 4;
  static constexpr int kRowWords = (OUT ? 2 * BN : BN) + 4;
  static constexpr int kRed = (kMaxKS - 1) * (128 / kMaxKS) * kRowWords * 4;
  static constexpr int kTok = 2 * BN * 4;                  // token scales (+ 256 x zero points)
  static constexpr int kFixed = kNP * (kPackA + kPackB) + kNO * (kOutA + kOutB) + kRed + kTok + 2048;
  // tensor memory: int32 accumulator, fp32 outlier accumulator, A stages
  static constexpr int kAcol = OUT ? 2 * BN : BN;
  static constexpr int kNWtmem = (512 - kAcol) / 64;        // 64-column stages (two K steps)
  static constexpr int kNWsmem = (kSmemBudget - kFixed) / kWideB;
  static constexpr int kNW = kNWtmem < kNWsmem ? (kNWtmem < 6 ? kNWtmem : 6)
                                               : (kNWsmem < 6 ? kNWsmem : 6);
  static constexpr int off_wide_b = 0;                     // 1024-aligned
  static constexpr int off_out_a = off_wide_b + kNW * kWideB;
  static constexpr int off_out_b = off_out_a + kNO * kOutA;
  static constexpr int off_pack_a = off_out_b + kNO * kOutB;
  static constexpr int off_pack_b = off_pack_a + kNP * kPackA;
  static constexpr int off_red = off_pack_b + kNP * kPackB;
  static constexpr int off_tok = off_red + kRed;
  static constexpr int off_bar = off_tok + kTok;
  // after the main loop the widened-stage area holds the epilogue staging:
  // the rows this CTA sends (int32 partials and outlier sums, kRowWords per
  // row), then the fp16 output box [tokens][owned rows] of the tensor store
  static constexpr int kSendBytes = (128 - 128 / kMaxKS) * kRowWords * 4;
  static constexpr int off_ybox = (kSendBytes + 1023) / 1024 * 1024;
  static_assert(off_ybox + BN * 128 * 2 <= kNW * kWideB, "epilogue staging");
  // full_p, empty_p, full_w, empty_w, full_o, empty_o, tmem_full, recv, drain,
  // rows_ready (fused kernel: the token rows of every CTA are in memory),
  // xbar[2] (fused kernel: the cluster's span maxima of a row landed)
  static constexpr int kNumBars = 2 * kNP + 2 * kNW + 2 * kNO + 6;
  static constexpr int off_misc = off_bar + 8 * kNumBars;
  // misc: TMEM base, abort flag, 8 spare bytes, then the fused kernel's
  // span maxima [2 row parities][max, -min][4 CTAs]
  static constexpr int off_xmax = off_misc + 16;
  static constexpr int kBytes = off_xmax + 64 + 1024;
  static_assert(kNW >= 3, "stage ring");
  static_assert(kBytes <= kSmemBudget, "shared memory");
  static_assert(BN == 32 || BN == 64, "token tile");
  static_assert(off_out_a % 1024 == 0 && off_out_b % 1024 == 0 && off_pack_a % 1024 == 0 &&
                    kPackB % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
};

// K steps of CTA `r` of a cluster of `ks`: int steps [i0, i1), outlier steps
// [o0, o1).  CTA 0 takes every outlier step and a share of the int steps
// that evens out the totals, an outlier step counting as 2/5 of an int step
// (its MMAs are short and its loads overlap the int ring); the other CTAs
// split the rest of the int steps.  Int ranges start at even steps (a ring
// slot holds two).
struct StepRange { int i0, i1, o0, o1; };

__device__ __forceinline__ StepRange step_range(int r, int ks, int kt, int ot) {
  StepRange s{0, kt, 0, ot};
  if (ks == 1) return s;
  const int per = (5 * kt + 2 * ot + 5 * ks - 1) / (5 * ks);
  const int first = min(kt, (max(0, per - (2 * ot + 4) / 5) + 1) & ~1);
  if (r == 0) return StepRange{0, first, 0, ot};
  const int q = (((kt - first + ks - 2) / (ks - 1)) + 1) & ~1;
  const int i0 = min(kt, first + (r - 1) * q);
  return StepRange{i0, min(kt, i0 + q), 0, 0};
}

// ------------------------------------------------------------ fused rotate

constexpr int kRotThreads = 384;          // warps 0-11 rotate before their GEMM roles
constexpr uint32_t kRotBar = 3;           // their named barrier

__device__ __forceinline__ void rot_sync() { named_barrier(kRotBar, kRotThreads); }

// Maximum over the rotating warps; `red` holds one float per warp.
__device__ __forceinline__ float rot_max(float v, float* red, int t) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((t & 31) == 0) red[t >> 5] = v;
  rot_sync();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kRotThreads / 32; ++w) m = fmaxf(m, red[w]);
  rot_sync();                              // red is reused
  return m;
}

// Position of span element e in the scatter buffer: one float of padding
// after every 16, so that threads writing 16 consecutive elements each hit
// distinct banks (17 is odd).
__device__ __forceinline__ int pad16(int e) { return e + (e >> 4); }

// The first butterfly pass of a span: groups of 8 consecutive elements read
// from the padded scatter buffer `pbuf`, R (<= 3) stages on index bits
// [0, R) in registers, written to `buf` in few_swz order with two 16-byte
// stores.  Returns the largest |value| this thread wrote.
template <int R>
__device__ __forceinline__ float wht_first_pass(const float* pbuf, float* buf, int nloc, int t) {
  float am = 0.0f;
  for (int g = t; g < (nloc >> 3); g += kRotThreads) {
    float x[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = pbuf[pad16(8 * g + k)];
#pragma unroll
    for (int st = 0; st < R; ++st)
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (!(k & (1 << st))) {
          const float a = x[k], b = x[k | (1 << st)];
          x[k] = a + b;
          x[k | (1 << st)] = a - b;
        }
#pragma unroll
    for (int k = 0; k < 8; ++k) am = fmaxf(am, fabsf(x[k]));
    *reinterpret_cast<float4*>(buf + few_swz(8 * g)) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4*>(buf + few_swz(8 * g) + 4) = make_float4(x[4], x[5], x[6], x[7]);
  }
  return am;
}

// Span of rotated positions [e_lo, e_hi) that CTA `rank` of a cluster of
// `ks` takes in every row: whole blocks (at least 128 positions), split as
// evenly as they go.  The host sizes the row buffer with the same rule.
__host__ __device__ __forceinline__ int fused_span(int Kp, int lb, int ks) {
  const int unit = (1 << lb) > 128 ? (1 << lb) : 128;
  return (Kp / unit + ks - 1) / ks * unit;
}

// Rotates and quantizes the token rows of this CTA's cluster (rows c, c + Q,
// ... below M for cluster c of Q) with the kRotThreads threads t.  Each row
// is split over the cluster's ks CTAs by fused_span; a CTA reads the source
// columns that can land in its span, keeps the non-outlier ones (one binary
// search of the ascending outlier list per thread, then a walk over its
// contiguous chunks), runs the butterflies on its span in shared memory
// (`buf`, few_swz order), and takes its span's absmax (or max and -max of
// -x).  The CTAs' maxima meet through distributed shared memory: each sends
// its maxima to every CTA of the cluster (`xmax`, two sets by row parity)
// and arrives on that CTA's `xbar`.  Codes always clamp to the quantizer's
// range (a no-op for codes in range).
template <bool ASYM>
__device__ void fused_rotate_rows(const FusedRows& f, int M, int rank, int ks, float* buf,
                                  float* pbuf, int* sidx, float* red, float* xmax, uint64_t* xbar,
                                  volatile int32_t* abort_flag, int32_t* status, int t) {
  const int cluster = static_cast<int>(blockIdx.x) / ks;
  const int nclusters = static_cast<int>(gridDim.x) / ks;
  if (cluster >= M) return;
  const int span = fused_span(f.Kp, f.lb, ks);
  const int e_lo = min(f.Kp, rank * span), e_hi = min(f.Kp, e_lo + span);
  const int nloc = e_hi - e_lo;
  // the source columns of [e_lo, e_hi) lie in [e_lo, e_hi + n_out)
  const int col_hi = min(f.K, e_hi + f.n_out);
  const int nch = nloc > 0 ? (col_hi - e_lo + 7) >> 3 : 0;
  const int cpt = (nch + kRotThreads - 1) / kRotThreads;     // contiguous chunks per thread
  for (int j = t; j < f.n_out; j += kRotThreads) sidx[j] = __ldg(f.outlier_idx + j);
  const int bm = (1 << f.lb) - 1;
  int it = 0;
  for (int row = cluster; row < M; row += nclusters, ++it) {
    const __half* srow = f.src + static_cast<int64_t>(row) * f.ld;
    uint4 raw[4];
    auto issue = [&](int q0) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col0 = e_lo + 8 * (t * cpt + q0 + q);
        raw[q] = make_uint4(0u, 0u, 0u, 0u);
        if (q0 + q < cpt && f.aligned && col0 + 8 <= f.K) raw[q] = ld_stream_v4(srow + col0);
      }
    };
    issue(0);                                // the loads' latency overlaps the work below
    rot_sync();                              // sidx staged; the last row's buf reads done
    if (rank == 0 && f.out16 != nullptr)
      for (int j = t; j < f.n_out; j += kRotThreads) {
        const int c = sidx[j];
        f.out16[static_cast<int64_t>(row) * f.n_out + j] =
            (c >= 0 && c < f.K) ? srow[c] : __float2half(0.0f);
      }
    for (int e = max(f.Kr, e_lo) + t; e < e_hi; e += kRotThreads) {
      if (f.padded) pbuf[pad16(e - e_lo)] = 0.0f;
      else buf[few_swz(e - e_lo)] = 0.0f;
    }
    for (int q0 = 0; q0 < cpt; q0 += 4) {
      if (q0 > 0) issue(q0);
      // outlier columns left of this batch's first column
      const int col_first = e_lo + 8 * (t * cpt + q0);
      int before = 0, hi = f.n_out;
      while (before < hi) {
        const int mid = (before + hi) >> 1;
        if (sidx[mid] < col_first) before = mid + 1;
        else hi = mid;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col0 = col_first + 8 * q;
        if (q0 + q >= cpt || col0 >= col_hi) break;
        float x[8];
        if (f.aligned && col0 + 8 <= f.K) {
          const __half2* h = reinterpret_cast<const __half2*>(&raw[q]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 v = __half22float2(h[i]);
            x[2 * i] = v.x;
            x[2 * i + 1] = v.y;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = (col0 + i < f.K) ? __half2float(srow[col0 + i]) : 0.0f;
        }
        uint32_t m8 = 0u;
        for (int k = before; k < f.n_out && k < before + 8; ++k) {
          const int d = sidx[k] - col0;
          if (d >= 8) break;
          if (d >= 0) m8 |= 1u << d;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = col0 + i - before;
          if ((m8 >> i) & 1u) {
            ++before;
          } else if (col0 + i < f.K && e < f.Kr && e >= e_lo && e < e_hi) {
            float xv = x[i];
            if (f.signs != nullptr && __ldg(f.signs + e) < 0) xv = -xv;
            if (f.padded) pbuf[pad16(e - e_lo)] = xv;
            else buf[few_swz(e - e_lo)] = xv;
          }
        }
      }
    }
    rot_sync();
    // stages [0, 3) (or all of a smaller block) on the way out of the
    // scatter buffer, the rest three at a time in place
    const int r0 = min(3, f.lb);
    float am = 0.0f;
    if (f.padded) {
      am = r0 == 3 ? wht_first_pass<3>(pbuf, buf, nloc, t)
         : r0 == 2 ? wht_first_pass<2>(pbuf, buf, nloc, t)
         : r0 == 1 ? wht_first_pass<1>(pbuf, buf, nloc, t)
                   : wht_first_pass<0>(pbuf, buf, nloc, t);
    } else {
      // (rows too long for both buffers: scattered straight into buf)
      am = r0 == 3 ? wht_smem_pass<3>(buf, nloc, 0, t, kRotThreads)
         : r0 == 2 ? wht_smem_pass<2>(buf, nloc, 0, t, kRotThreads)
         : r0 == 1 ? wht_smem_pass<1>(buf, nloc, 0, t, kRotThreads)
                   : 0.0f;
      if (r0 == 0)
        for (int e = t; e < nloc; e += kRotThreads) am = fmaxf(am, fabsf(buf[e]));
    }
    rot_sync();
    for (int s = 3; s < f.lb; s += 3) {
      const int r = min(3, f.lb - s);
      if (r == 3) am = wht_smem_pass<3>(buf, nloc, s, t, kRotThreads);
      else if (r == 2) am = wht_smem_pass<2>(buf, nloc, s, t, kRotThreads);
      else am = wht_smem_pass<1>(buf, nloc, s, t, kRotThreads);
      rot_sync();
    }
    float m0 = am, m1 = 0.0f;
    if (ASYM) {
      m0 = -INFINITY;
      m1 = -INFINITY;
      for (int e = t; e < nloc; e += kRotThreads) {
        m0 = fmaxf(m0, buf[e]);
        m1 = fmaxf(m1, -buf[e]);
      }
      m1 = rot_max(m1, red, t);
    }
    m0 = rot_max(m0, red, t);
    if (ks > 1) {
      // every CTA's maxima into every CTA of the cluster, then wait for all
      const int par = it & 1;
      if (t < ks) {
        const uint32_t dst = mapa_shared(smem_u32(xmax + 8 * par + rank), static_cast<uint32_t>(t));
        asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst), "f"(m0) : "memory");
        if (ASYM) asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst + 16u), "f"(m1) : "memory");
        mbar_arrive_cluster(mapa_shared(smem_u32(xbar + par), static_cast<uint32_t>(t)));
      }
      mbar_wait_cluster_bounded(xbar + par, static_cast<uint32_t>((it >> 1) & 1), abort_flag, status,
                                kDevTimeoutGridSync);
      for (int i = 0; i < ks; ++i) {
        m0 = fmaxf(m0, xmax[8 * par + i]);
        if (ASYM) m1 = fmaxf(m1, xmax[8 * par + 4 + i]);
      }
    }
    const bool lead = t == 0 && rank == 0;
    const RowQ q = ASYM ? asym_row_q(-m1, m0, f.clip_ratio, f.inv_sqrt_block,
                                     lead ? f.scales + row : nullptr, f.zeros + row)
                        : sym_row_q(m0, f.clip_ratio, f.inv_sqrt_block,
                                    lead ? f.scales + row : nullptr);
    uint8_t* crow = f.codes + static_cast<int64_t>(row) * (f.Kp >> 1) + (e_lo >> 1);
    for (int g = t; g < (nloc >> 3); g += kRotThreads) {
      const int el = 8 * g;
      float v[8];
      if (f.gsr) {
        // sequency position j of a block takes Hadamard output bitrev(gray(j))
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = (el + i) & bm;
          const int nat = static_cast<int>(__brev(static_cast<unsigned>(j ^ (j >> 1))) >> (32 - f.lb));
          v[i] = buf[few_swz(((el + i) & ~bm) + nat)];
        }
      } else {
        const float4 a = *reinterpret_cast<const float4*>(buf + few_swz(el));
        const float4 b = *reinterpret_cast<const float4*>(buf + few_swz(el) + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      }
      *reinterpret_cast<uint32_t*>(crow + (el >> 1)) = quant_word<true>(v, q.r, q.c, q.lo, q.hi);
    }
  }
}

template <int BN, bool OUT, bool ASYM, bool ROT>
__global__ void __launch_bounds__(kThreads, 1)
w4a4_gemm_decode_kernel(const __grid_constant__ CUtensorMap map_w,
                        const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_wo,
                        const __grid_constant__ CUtensorMap map_xo,
                        const __grid_constant__ CUtensorMap map_y, const DecodeParams p) {
  using L = DecodeLayout<BN, OUT>;
  constexpr int kNW = L::kNW;
  constexpr uint32_t kAcol = L::kAcol;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* full_p = bars;                   // TMA landed
  uint64_t* empty_p = full_p + kNP;          // widen group done reading (4 warps)
  uint64_t* full_w = empty_p + kNP;          // stage widened (4 warps)
  uint64_t* empty_w = full_w + kNW;          // MMAs done with the stage
  uint64_t* full_o = empty_w + kNW;          // outlier TMA landed
  uint64_t* empty_o = full_o + kNO;          // MMAs done with the outlier stage
  uint64_t* tmem_full = empty_o + kNO;       // accumulators final
  uint64_t* recv = tmem_full + 1;            // the other CTAs' partials of my rows landed
  uint64_t* drain = recv + 1;
  uint64_t* rows_ready = drain + 1;          // fused: every CTA's token rows are in memory
  uint64_t* xbar = rows_ready + 1;           // fused: [2] the cluster's row maxima landed
  float* xmax = reinterpret_cast<float*>(smem + L::off_xmax);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::off_misc);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + L::off_misc + 4);
  uint32_t* slots = reinterpret_cast<uint32_t*>(smem + L::off_red);
  const int own_rows = 128 / p.ks;           // tile rows this CTA finishes

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = p.ks > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int tile = blockIdx.x / p.ks;
  const StepRange sr = step_range(rank, p.ks, p.kt, p.ot);
  const int n_int = sr.i1 - sr.i0, n_out = OUT ? sr.o1 - sr.o0 : 0;
  const int n_slots = (n_int + 1) >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNP; ++i) { mbar_init(&full_p[i], 1); mbar_init(&empty_p[i], 4); }
    for (int i = 0; i < kNW; ++i) { mbar_init(&full_w[i], 4); mbar_init(&empty_w[i], 1); }
    for (int i = 0; i < kNO; ++i) { mbar_init(&full_o[i], 1); mbar_init(&empty_o[i], 1); }
    mbar_init(tmem_full, 1);
    mbar_init(recv, 1);
    mbar_init(drain, 1);
    mbar_init(rows_ready, 1);
    mbar_init(&xbar[0], static_cast<uint32_t>(p.ks));
    mbar_init(&xbar[1], static_cast<uint32_t>(p.ks));
    *abort_flag = 0;
    fence_mbar_init();
    // the other CTAs' partials of my rows arrive by bulk copies
    if (p.ks > 1)
      mbar_arrive_expect_tx(recv, static_cast<uint32_t>((p.ks - 1) * own_rows * L::kRowWords * 4));
  }
  if (warp == kProducerWarp && lane == 0) {
    if (n_int > 0) { tma_prefetch_desc(&map_w); tma_prefetch_desc(&map_x); }
    if (n_out > 0) { tma_prefetch_desc(&map_wo); tma_prefetch_desc(&map_xo); }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (p.ks > 1) cluster_sync();              // every CTA's barriers initialized
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();                           // the previous kernel's outputs are visible
  grid_dep_launch();
  const int y_w = tile * 128;                // first weight row of the tile

  if (ROT && warp < kRotThreads / 32) {
    // ------------------------------------------------------------ fused rotate
    // the wide-B area is free until these warps start widening
    float* rbuf = reinterpret_cast<float*>(smem + L::off_wide_b);
    const int span = fused_span(p.rows.Kp, p.rows.lb, p.ks);
    float* pbuf = rbuf + span;
    int* ridx = reinterpret_cast<int*>(p.rows.padded ? pbuf + pad16(span) : pbuf);
    float* rred = reinterpret_cast<float*>(ridx + p.rows.n_out);
    fused_rotate_rows<ASYM>(p.rows, p.M, rank, p.ks, rbuf, pbuf, ridx, rred, xmax, xbar,
                            abort_flag, p.status, static_cast<int>(threadIdx.x));
    __threadfence();                         // this CTA's rows, visible GPU-wide
    fence_proxy_async_global();
    rot_sync();
    if (threadIdx.x == 0) {
      grid_sync_bounded(p.rows.sync, gridDim.x, p.status);
      mbar_arrive(rows_ready);
    }
  }

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0;
      if (ROT) {
        // the weight halves of the first slots go out before the token rows
        // exist; their token halves follow the grid barrier
        const uint32_t pre = static_cast<uint32_t>(min(kNP, n_slots));
        for (uint32_t i = 0; i < pre; ++i) {
          mbar_arrive_expect_tx(&full_p[i], L::kPackA + L::kPackB);
          tma_load_2d(smem + L::off_pack_a + i * L::kPackA, &map_w, &full_p[i],
                      (sr.i0 + 2 * static_cast<int>(i)) * kStep, y_w);
        }
        ok = mbar_wait_bounded(rows_ready, 0, abort_flag, p.status, kDevTimeoutProducer);
        fence_proxy_async_global();
        // (issued even after a timeout, so that every slot completes)
        for (uint32_t i = 0; i < pre; ++i)
          tma_load_2d(smem + L::off_pack_b + i * L::kPackB, &map_x, &full_p[i],
                      (sr.i0 + 2 * static_cast<int>(i)) * kStep, 0);
        it = pre;
      }
      for (; static_cast<int>(it) < n_slots; ++it) {
        const uint32_t s = it % kNP, ph = (it / kNP) & 1;
        const int x = (sr.i0 + 2 * static_cast<int>(it)) * kStep;
        if (!(ok = mbar_wait_bounded(&empty_p[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
        mbar_arrive_expect_tx(&full_p[s], L::kPackA + L::kPackB);
        tma_load_2d(smem + L::off_pack_a + s * L::kPackA, &map_w, &full_p[s], x, y_w);
        tma_load_2d(smem + L::off_pack_b + s * L::kPackB, &map_x, &full_p[s], x, 0);
      }
      if (!ok)
        for (uint32_t i = (it > kNP ? it - kNP : 0); i < it; ++i)
          mbar_wait_bounded(&full_p[i % kNP], (i / kNP) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
    } else if (OUT && lane == 1 && n_out > 0) {
      // the outlier ring, beside the int ring, so that its loads overlap it
      bool ok = true;
      uint32_t ot = 0;
      if (ROT) {
        ok = mbar_wait_bounded(rows_ready, 0, abort_flag, p.status, kDevTimeoutProducer);
        fence_proxy_async_global();
      }
      for (int os = sr.o0; os < sr.o1; ++os, ++ot) {
        const uint32_t s = ot % kNO, ph = (ot / kNO) & 1;
        if (!(ok = mbar_wait_bounded(&empty_o[s], ph ^ 1, abort_flag, p.status, kDevTimeoutProducer))) break;
        mbar_arrive_expect_tx(&full_o[s], L::kOutA + L::kOutB);
        tma_load_2d(smem + L::off_out_a + s * L::kOutA, &map_wo, &full_o[s], os * kOutCols, y_w);
        tma_load_2d(smem + L::off_out_b + s * L::kOutB, &map_xo, &full_o[s], os * kOutCols, 0);
      }
      if (!ok)
        for (uint32_t i = (ot > kNO ? ot - kNO : 0); i < ot; ++i)
          mbar_wait_bounded(&full_o[i % kNO], (i / kNO) & 1, abort_flag, nullptr, 0, kDrainLimitNs);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BN);
      constexpr uint32_t idesc_o = idesc_f16(BN);
      bool ok = true;
      int ot = 0;                                // outlier steps done
      // one fp16 outlier step (two K16 MMAs into the fp32 accumulator)
      auto outlier_step = [&]() {
        const uint32_t s = ot % kNO, ph = (ot / kNO) & 1;
        if (!(ok = mbar_wait_bounded(&full_o[s], ph, abort_flag, p.status, kDevTimeoutMma))) return;
        tc_fence_after();
        const uint64_t da = smem_desc_kmajor(smem_u32(smem + L::off_out_a + s * L::kOutA), 64);
        const uint64_t db = smem_desc_kmajor(smem_u32(smem + L::off_out_b + s * L::kOutB), 64);
#pragma unroll
        for (int k = 0; k < 2; ++k) mma_f16(tmem_base + BN, da + 2 * k, db + 2 * k, idesc_o, (ot | k) != 0);
        mma_commit(&empty_o[s]);
        ++ot;
      };
      for (int it = 0; it < n_slots; ++it) {
        const uint32_t s = it % kNW, ph = (it / kNW) & 1;
        if (!(ok = mbar_wait_bounded(&full_w[s], ph, abort_flag, p.status, kDevTimeoutMma))) break;
        tc_fence_after();
        // two K steps; past this CTA's range (odd count) both operands are
        // zero-filled or, inside K, a step another CTA also takes: skip it
        const int nk = (2 * it + 1 < n_int) ? 8 : 4;
        const uint32_t a = tmem_base + kAcol + s * 64;
        const uint64_t db0 = smem_desc_kmajor(smem_u32(smem + L::off_wide_b + s * L::kWideB), 128);
        const uint64_t db1 = smem_desc_kmajor(smem_u32(smem + L::off_wide_b + s * L::kWideB + L::kWideBlk), 128);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k < nk) mma_i8_ts(tmem_base, a + 8 * k, (k < 4 ? db0 : db1) + 2 * (k & 3), idesc, (it | k) != 0);
        mma_commit(&empty_w[s]);
        if (OUT && it >= 1 && ot < n_out) {
          outlier_step();
          if (!ok) break;
        }
      }
      if (OUT)
        while (ok && ot < n_out) outlier_step();
      if (ok) mma_commit(tmem_full);
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, abort_flag, p.status, kDevTimeoutDrain, kDrainLimitNs);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ widen
    const int wt = threadIdx.x - 128;
    const int group = wt >> 7;                     // takes the ring slots it with it % 2 == group
    const int row = wt & 127;                      // weight row of the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    for (int it = group; it < n_slots && ok; it += 2) {
      const uint32_t s = it % kNP, ph = (it / kNP) & 1;
      const uint32_t sw = it % kNW, phw = (it / kNW) & 1;
      if (!(ok = mbar_wait_bounded(&full_p[s], ph, abort_flag, p.status, kDevTimeoutWiden))) break;
      if (!(ok = mbar_wait_bounded(&empty_w[sw], phw ^ 1, abort_flag, p.status, kDevTimeoutWiden))) break;
      {
        // weight row: 128 packed bytes (128-byte swizzled rows) -> 256 s8 in TMEM
        const uint8_t* pa = smem + L::off_pack_a + s * L::kPackA + row * kSlot;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(pa + (((4 * h + c) ^ (row & 7)) << 4));
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
      {
        // token rows (128-byte swizzled): each 16-byte packed chunk -> two
        // 16-byte s8 chunks of the K block it belongs to, SW128
        const uint8_t* pb = smem + L::off_pack_b + s * L::kPackB;
        uint8_t* wb = smem + L::off_wide_b + sw * L::kWideB;
        for (int task = row; task < BN * 4; task += 128) {
          const int br = task >> 2, c = task & 3;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint4 u = *reinterpret_cast<const uint4*>(pb + br * kSlot + (((4 * h + c) ^ (br & 7)) << 4));
            uint4 ev, od;
            ev.x = (u.x << 4) & 0xF0F0F0F0u; od.x = u.x & 0xF0F0F0F0u;
            ev.y = (u.y << 4) & 0xF0F0F0F0u; od.y = u.y & 0xF0F0F0F0u;
            ev.z = (u.z << 4) & 0xF0F0F0F0u; od.z = u.z & 0xF0F0F0F0u;
            ev.w = (u.w << 4) & 0xF0F0F0F0u; od.w = u.w & 0xF0F0F0F0u;
            uint8_t* base = wb + h * L::kWideBlk + (br >> 3) * 1024 + (br & 7) * 128;
            *reinterpret_cast<uint4*>(base + (((2 * c) ^ (br & 7)) << 4)) = ev;
            *reinterpret_cast<uint4*>(base + (((2 * c + 1) ^ (br & 7)) << 4)) = od;
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
  } else {
    // ------------------------------------------------------------ epilogue
    // Lane = tile row (output column n).  Rows another CTA owns: the int32
    // partials (and CTA 0's fp32 outlier sums) are staged in this CTA's
    // shared memory and sent with one bulk copy per warp into the owner's
    // receive slot.  Owned rows: partials added, dequantized with the token
    // scales staged in shared memory, written as fp16 into a [token][row]
    // box that one thread hands to a tensor store.
    const int lrow = warp * 32 + lane;             // tile row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int owner = lrow / own_rows;             // the CTA that finishes this row
    const bool has_out = OUT && p.ot > 0;
    const int n = y_w + lrow;                      // output column = weight row
    float* tok = reinterpret_cast<float*>(smem + L::off_tok);   // [BN] scales, [BN] 256 x zeros
    if (warp == 0) {
      if (ROT) {
        // written in this launch by other CTAs: after the grid barrier, and
        // through L2 (not the read-only path)
        mbar_wait_bounded(rows_ready, 0, abort_flag, p.status, kDevTimeoutEpilogue);
        for (int i = lane; i < BN; i += 32) {
          tok[i] = i < p.M ? __ldcg(p.a_scales + i) : 0.0f;
          if (ASYM) tok[BN + i] = i < p.M ? 256.0f * static_cast<float>(__ldcg(p.a_zeros + i)) : 0.0f;
        }
      } else {
        for (int i = lane; i < BN; i += 32) {
          tok[i] = i < p.M ? __ldg(p.a_scales + i) : 0.0f;
          if (ASYM) tok[BN + i] = i < p.M ? 256.0f * static_cast<float>(__ldg(p.a_zeros + i)) : 0.0f;
        }
      }
    }
    named_barrier(1, 128);                         // the four epilogue warps
    // asymmetric activations: acc - 256 * zero[m] * w_sum[n] (the accumulator is 256 x)
    float s_row = 0.0f, wsum = 0.0f;
    if (owner == rank && n < p.N) {
      s_row = __ldg(p.w_scales + n) * (1.0f / 256.0f);
      if (ASYM) wsum = static_cast<float>(__ldg(p.w_sums + n));
    }
    bool ok = mbar_wait_bounded(tmem_full, 0, abort_flag, p.status, kDevTimeoutEpilogue);
    tc_fence_after();
    if (owner != rank) {
      // rows sent, in order: all rows but the owned block
      const int srow = lrow < rank * own_rows ? lrow : lrow - own_rows;
      uint32_t* stg = reinterpret_cast<uint32_t*>(smem + L::off_wide_b) + srow * L::kRowWords;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t acc[32];
        tmem_ld_32x32b_x32(tmem_base + lane_off + c * 32, acc);
        tmem_ld_wait();
        const bool zero = n_int == 0 || !ok;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(stg + c * 32 + 4 * q) =
              zero ? make_uint4(0u, 0u, 0u, 0u)
                   : make_uint4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        if (has_out && rank == 0) {
          tmem_ld_32x32b_x32(tmem_base + lane_off + BN + c * 32, acc);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(stg + BN + c * 32 + 4 * q) =
                make_uint4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // this warp's 32 rows are contiguous both here and in the owner's slot
        const int slot = (rank - owner - 1 + p.ks) % p.ks;
        const uint32_t dst = mapa_shared(smem_u32(slots), static_cast<uint32_t>(owner)) +
                             4u * static_cast<uint32_t>((slot * own_rows + lrow % own_rows) * L::kRowWords);
        bulk_copy_to_cluster(dst, stg, 32u * L::kRowWords * 4u,
                             mapa_shared(smem_u32(recv), static_cast<uint32_t>(owner)));
      }
    } else {
      // finish this row: own partial + the received ones, dequantize, store
      if (p.ks > 1) {
        const bool got = mbar_wait_cluster_bounded(recv, 0, abort_flag, p.status, kDevTimeoutEpilogue);
        ok = ok && got;
      }
      const bool n_ok = ok && n < p.N;
      const int r_local = lrow % own_rows;
      const int slot0 = (0 - rank - 1 + p.ks) % p.ks;   // CTA 0's slot (outlier sums)
      __half* ybox = reinterpret_cast<__half*>(smem + L::off_wide_b + L::off_ybox);
      const float4* tok4 = reinterpret_cast<const float4*>(tok);
      const float4* zer4 = reinterpret_cast<const float4*>(tok + BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t acc[32];
        uint32_t oacc[32];
        tmem_ld_32x32b_x32(tmem_base + lane_off + c * 32, acc);
        if (OUT) tmem_ld_32x32b_x32(tmem_base + lane_off + BN + c * 32, oacc);
        tmem_ld_wait();
        if (n_int == 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[j] = 0;
        }
        for (int sl = 0; sl < p.ks - 1; ++sl) {
          const uint4* src = reinterpret_cast<const uint4*>(
              slots + (sl * own_rows + r_local) * L::kRowWords + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 v = src[q];
            acc[4 * q] += v.x; acc[4 * q + 1] += v.y; acc[4 * q + 2] += v.z; acc[4 * q + 3] += v.w;
          }
        }
        if (OUT && has_out && rank != 0) {
          const uint4* src = reinterpret_cast<const uint4*>(
              slots + (slot0 * own_rows + r_local) * L::kRowWords + BN + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 v = src[q];
            oacc[4 * q] = v.x; oacc[4 * q + 1] = v.y; oacc[4 * q + 2] = v.z; oacc[4 * q + 3] = v.w;
          }
        }
        // dequantize all 32 tokens first (no branches: independent chains),
        // then store them
        uint32_t hp[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 sa4 = tok4[c * 8 + q];
          const float sav[4] = {sa4.x, sa4.y, sa4.z, sa4.w};
          float zav[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          if (ASYM) {
            const float4 z4 = zer4[c * 8 + q];
            zav[0] = z4.x; zav[1] = z4.y; zav[2] = z4.z; zav[3] = z4.w;
          }
          float y[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int j = 4 * q + t;
            float af = static_cast<float>(static_cast<int32_t>(acc[j]));
            if (ASYM) af = fmaf(-zav[t], wsum, af);
            y[t] = af * s_row * sav[t];
            if (has_out) y[t] += __uint_as_float(oacc[j]);
          }
          const __half2 h0 = __floats2half2_rn(y[0], y[1]);
          const __half2 h1 = __floats2half2_rn(y[2], y[3]);
          hp[2 * q] = *reinterpret_cast<const uint32_t*>(&h0);
          hp[2 * q + 1] = *reinterpret_cast<const uint32_t*>(&h1);
        }
        if (p.y_tma) {
          uint16_t* yb = reinterpret_cast<uint16_t*>(ybox) + c * 32 * own_rows + r_local;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            yb[j * own_rows] = static_cast<uint16_t>(hp[j / 2] >> (16 * (j & 1)));
        } else if (n_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j < p.M)
              reinterpret_cast<uint16_t*>(p.Y)[static_cast<int64_t>(c * 32 + j) * p.ldy + n] =
                  static_cast<uint16_t>(hp[j / 2] >> (16 * (j & 1)));
        }
        if (p.acc_debug != nullptr && n_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j < p.M)
              p.acc_debug[static_cast<int64_t>(c * 32 + j) * p.N + n] = static_cast<int32_t>(acc[j]) >> 8;
        }
      }
      if (p.y_tma) {
        // rows past N and tokens past M fall outside the tensor: not written
        fence_proxy_async_smem();
        named_barrier(2, static_cast<uint32_t>(own_rows));   // the owner warps
        if (r_local == 0) {
          if (ok) {
            tma_store_2d(&map_y, ybox, y_w + rank * own_rows, 0);
            bulk_commit_group();
          }
          bulk_wait_group<0>();
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (p.ks > 1) cluster_sync();              // no CTA leaves while another may still signal it
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int BN, bool OUT, bool ASYM, bool ROT>
cudaError_t run_decode(const CUtensorMap& mw, const CUtensorMap& mx, const CUtensorMap& mwo,
                       const CUtensorMap& mxo, const CUtensorMap& my, const DecodeParams& p,
                       int tiles, cudaStream_t stream) {
  auto k = w4a4_gemm_decode_kernel<BN, OUT, ASYM, ROT>;
  const int smem = DecodeLayout<BN, OUT>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(tiles * p.ks);
  if (!ROT) {
    e = launch_pdl(k, dim3(grid), dim3(kThreads), smem, stream, static_cast<unsigned>(p.ks), mw, mx,
                   mwo, mxo, my, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  // The fused kernel's CTAs meet at a grid-wide barrier, so all of them must
  // be resident at once: the launch goes ahead only when every cluster fits
  // on the device together.  It keeps programmatic dependent launch: CTAs
  // that start early wait in grid_dep_wait until the previous kernel has
  // finished, and the rest start as that kernel's CTAs leave, so all of them
  // become resident; the barrier's bounded wait guards the rest (another
  // process holding SMs).
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  int64_t resident = 0;
  if (p.ks > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(p.ks);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
    cfg.attrs = attr;
    cfg.numAttrs = n;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, k, &cfg);
    if (e != cudaSuccess) return e;
    resident = static_cast<int64_t>(clusters) * p.ks;
  } else {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, smem);
    if (e != cudaSuccess) return e;
    resident = static_cast<int64_t>(per_sm) * sm_count();
  }
  if (resident < static_cast<int64_t>(grid)) return cudaErrorCooperativeLaunchTooLarge;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = n + 1;
  e = cudaLaunchKernelEx(&cfg, k, mw, mx, mwo, mxo, my, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

// CTAs per cluster splitting K: the largest of 1, 2, 4 with tiles x KS <= SMs
// and at least one K step per CTA.
int decode_k_split(int64_t tiles, int64_t steps, int sms) {
  int ks = 1;
  while (ks < 4 && tiles * ks * 2 <= sms && steps >= ks * 2) ks *= 2;
  return ks;
}

namespace {

qr_status decode_common(const GemmJob& j, const FusedRows* fr, cudaStream_t stream) {
  const bool out = j.n_out > 0;
  const int bn = j.M <= 32 ? 32 : 64;
  const int64_t tiles = (j.N + 127) / 128;
  DecodeParams p{};
  p.w_scales = j.w_scales;
  p.a_scales = j.a_scales;
  p.a_zeros = j.a_zeros;
  p.w_sums = j.w_sums;
  p.Y = reinterpret_cast<__half*>(j.Y);
  p.ldy = j.ldy;
  p.acc_debug = j.acc_debug;
  p.N = static_cast<int32_t>(j.N);
  p.M = static_cast<int32_t>(j.M);
  p.kt = static_cast<int32_t>(j.Kp / 128);
  p.ot = out ? (j.n_out + kOutCols - 1) / kOutCols : 0;
  p.ks = std::min(decode_k_split(tiles, p.kt + p.ot, sm_count()), bn == 64 ? 2 : 4);
  // Y through tensor stores: per owner block, a box of (128 / KS) rows x BN tokens
  CUtensorMap my{};
  p.y_tma = (reinterpret_cast<uintptr_t>(j.Y) % 16 == 0) && (j.ldy % 8 == 0) &&
            make_tensor_map_2d(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.Y, static_cast<uint64_t>(j.N),
                               static_cast<uint64_t>(j.M), static_cast<uint64_t>(j.ldy) * 2,
                               static_cast<uint32_t>(128 / p.ks), static_cast<uint32_t>(bn),
                               CU_TENSOR_MAP_SWIZZLE_NONE);
  p.status = device_status_word();
  if (p.status == nullptr) return QR_ERR_CUDA;
  CUtensorMap mw{}, mx{}, mwo{}, mxo{};
  const uint64_t kb = static_cast<uint64_t>(j.Kp) / 2;   // packed bytes per row
  if (p.kt > 0 &&
      (!make_tensor_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.w_codes, kb, j.N, kb, kSlot, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
       !make_tensor_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, j.a_codes, kb, j.M, kb, kSlot, bn,
                           CU_TENSOR_MAP_SWIZZLE_128B)))
    return QR_ERR_CUDA;
  if (out) {
    const uint64_t no = static_cast<uint64_t>(j.n_out);
    if (!make_tensor_map_2d(&mwo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.w_out, no, j.N, no * 2,
                            kOutCols, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_tensor_map_2d(&mxo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, j.x_out, no, j.M, no * 2,
                            kOutCols, bn, CU_TENSOR_MAP_SWIZZLE_64B))
      return QR_ERR_CUDA;
  }
  const int t = static_cast<int>(tiles);
  cudaError_t e;
  const bool asym = p.a_zeros != nullptr;
  if (fr != nullptr) {
    p.rows = *fr;
    // the row buffer, the padded scatter buffer (when there is room), the
    // outlier list and the warp maxima live in the wide-B area until the
    // ring starts
    const int span = fused_span(fr->Kp, fr->lb, p.ks);
    const int64_t need = 4ll * (span + fr->n_out + kRotThreads / 32);
    const int64_t pad_need = need + 4ll * (span + span / 16);
    const int64_t room = bn == 32 ? (out ? DecodeLayout<32, true>::kNW * DecodeLayout<32, true>::kWideB
                                         : DecodeLayout<32, false>::kNW * DecodeLayout<32, false>::kWideB)
                                  : (out ? DecodeLayout<64, true>::kNW * DecodeLayout<64, true>::kWideB
                                         : DecodeLayout<64, false>::kNW * DecodeLayout<64, false>::kWideB);
    if (need > room) return QR_ERR_UNSUPPORTED;
    p.rows.padded = pad_need <= room;
  }
  const bool rot = fr != nullptr;
#define QR_RUN_DECODE(B, O)                                                                  \
  (rot ? (asym ? run_decode<B, O, true, true>(mw, mx, mwo, mxo, my, p, t, stream)            \
               : run_decode<B, O, false, true>(mw, mx, mwo, mxo, my, p, t, stream))          \
       : (asym ? run_decode<B, O, true, false>(mw, mx, mwo, mxo, my, p, t, stream)           \
               : run_decode<B, O, false, false>(mw, mx, mwo, mxo, my, p, t, stream)))
  if (bn == 32) e = out ? QR_RUN_DECODE(32, true) : QR_RUN_DECODE(32, false);
  else e = out ? QR_RUN_DECODE(64, true) : QR_RUN_DECODE(64, false);
#undef QR_RUN_DECODE
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return QR_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace

qr_status launch_w4a4_gemm_decode(const GemmJob& j, cudaStream_t stream) {
  return decode_common(j, nullptr, stream);
}

qr_status launch_w4a4_decode_fused(const GemmJob& j, const RowJob& r, uint32_t* sync,
                                   cudaStream_t stream) {
  const qr_rotation& rot = *r.rot;
  if (rot.kind != QR_ROT_NONE && rot.kind != QR_ROT_HADAMARD && rot.kind != QR_ROT_GSR)
    return QR_ERR_UNSUPPORTED;
  if (j.M > 64 || r.rows != j.M || r.Kp != j.Kp || r.n_out != j.n_out) return QR_ERR_INVALID_ARG;
  FusedRows f{};
  f.src = reinterpret_cast<const __half*>(r.src);
  f.ld = r.ld;
  f.K = static_cast<int32_t>(r.K);
  f.Kr = r.Kr;
  f.Kp = r.Kp;
  f.n_out = r.n_out;
  f.outlier_idx = r.outlier_idx;
  f.signs = rot.kind == QR_ROT_NONE ? nullptr : rot.signs;
  const int block = rot.kind == QR_ROT_NONE ? 1 : rot.block;
  int lb = 0;
  while ((1 << lb) < block) ++lb;
  f.lb = lb;
  f.gsr = rot.kind == QR_ROT_GSR;
  f.aligned = (reinterpret_cast<uintptr_t>(r.src) % 16 == 0) && (r.ld % 8 == 0);
  f.clip_ratio = rot.clip_ratio;
  f.inv_sqrt_block = static_cast<float>(1.0 / std::sqrt(static_cast<double>(block)));
  f.codes = r.codes;
  f.scales = r.scales;
  f.zeros = r.zeros;
  f.out16 = reinterpret_cast<__half*>(r.out16);
  f.sync = sync;
  return decode_common(j, &f, stream);
}



}  // namespace qr
