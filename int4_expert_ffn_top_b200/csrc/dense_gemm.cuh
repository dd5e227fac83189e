// Dense tcgen05 GEMMs over the layer input u (bf16 [T][H]) for many-token batches.
//
//  * The 8-bit router (MODE_ROUTER): logits[t][e] = sum_g (s_eg D_eg(t) + b'_eg U_g(t)) + beta_e, where
//    D_eg(t) = sum_{k in group g} (q_ek - 128) u_tk is one quantisation group's tensor-core product, U_g(t) =
//    sum_{k in g} u_tk, and b'_eg = b_eg + 128 s_eg: the affine group-64 weight w = q s + b split as
//    s (q - 128) + b'.  Codes minus 128 and bf16 activations are both bf16 values, so every product is exact;
//    each group accumulates into its own TMEM accumulator, which the epilogue scales and folds into fp32
//    registers, so no dequantised weight is ever rounded.
//  * The Prerouter's first layer (MODE_W1): z[t][p] = silu(sum_k W1[p][k] x_t[k] + b1[p]) over the input
//    x_t = [u_t ; m_t], m_t the multi-hot of the token's executed experts.  The fp16 W1 is split exactly into
//    two bf16 parts (hi = bf16(w) and lo = w - hi, which has at most three significant bits), both multiplied
//    with the bf16 operand, so no input is rounded either; the multi-hot part of the token operand is built in
//    shared memory (the last E/64 K steps).
//
// A tile is 128 output rows (experts, Prerouter units) x 64 tokens; K advances 64 per step.  One CTA per SM
// walks the tiles (c, c + grid, ...) with every role running the same (tile, step) sequence:
//  * warp 0, one lane (TMA): the raw A rows (router: 128 code bytes = two steps per copy; W1: 64 fp16 = one
//    step) and the step's 64 token rows of u, both 128-byte swizzled; rows past T read as zeros;
//  * warps 1, 2, one lane each (MMA; one thread issues an MMA only every ~175 cycles): tcgen05.mma kind::f16
//    with bf16 operands into fp32 TMEM accumulators -- router: the group's four 16-wide K slices into
//    accumulator b = step % 4, issued by MMA warp b % 2; W1: slice c of every step (hi then lo) into chain c,
//    chains split over the MMA warps, two tiles in flight;
//  * 8 converting warps: raw rows -> bf16 operand stage(s) in the 128-byte-swizzled K-major layout the MMA
//    reads; router: also U_g of the step's 64 token rows (four lanes per token), handed to the epilogue in
//    shared memory; W1: the multi-hot token rows of the last E/64 steps;
//  * 8 epilogue warps (TMEM lane quadrant = warp % 4, two warps per quadrant, 32 token columns each): router:
//    per group, acc = fma(s, D, acc), acc = fma(b', U, acc), then + beta; W1: the sum of the four chains, + b1,
//    SiLU.  Outputs are fp32 rows [T][rows]: lanes = consecutive rows, one coalesced 128-byte store per token.
// Every wait is bounded; a role whose wait runs out stops issuing, lets what it issued land (bounded) and
// records MOE_ERR_TIMEOUT.
#pragma once

#include <cuda_bf16.h>

#include "tc_primitives.cuh"

namespace moe {
namespace dense {

using tc::bar_arrive;
using tc::bar_expect_tx;
using tc::bar_init;
using tc::bar_wait;
using tc::mma_commit;
using tc::mma_f16;
using tc::sa;
using tc::smem_desc;
using tc::tma_load_2d;
using tc::tmem_ld32;

enum Mode { MODE_ROUTER = 0, MODE_W1 = 1 };

constexpr int BM = 128;
constexpr int BN = 64;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int RSTAGES = 3;
constexpr int NACC = 4;  // router: group accumulators in flight
constexpr int kCvtWarps = 8;
constexpr int kEpiWarps = 8;
constexpr int A_SUB = BM * BK * 2;    // one bf16 operand stage, 16 KB
constexpr int B_STAGE = BN * BK * 2;  // 8 KB
constexpr int RAW_STAGE = BM * 128;   // 128 bytes per row, 16 KB

template <int MODE>
struct Cfg {
  static constexpr bool kRouter = MODE == MODE_ROUTER;
  static constexpr int kMma = 2;  // MMA-issuing warps: one thread issues an MMA only every ~175 cycles
  static constexpr int RAW_STEPS = kRouter ? 2 : 1;        // K steps per raw copy
  static constexpr int A_STAGE = kRouter ? A_SUB : 2 * A_SUB;  // W1: hi and lo parts
  static constexpr int kThreads = 32 * (1 + kMma + kCvtWarps + kEpiWarps);
  static constexpr int kWarpCvt0 = 1 + kMma;
  static constexpr int kWarpEpi0 = kWarpCvt0 + kCvtWarps;
  static constexpr int NA = kRouter ? NACC : 2;            // accumulator buffers (router: groups; W1: tiles)
  static constexpr uint32_t TMEM_COLS = kRouter ? NACC * BN : 2 * 4 * BN;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
  static constexpr int OFF_RAW = OFF_B + STAGES * B_STAGE;
  static constexpr int OFF_U = OFF_RAW + RSTAGES * RAW_STAGE;
  static constexpr int OFF_SB = OFF_U + (kRouter ? NACC * BN * 4 : 0);
  // router: each epilogue warp's copy of its 32 rows' scales and biases, H/64 + 1 words per row (the extra
  // word keeps the rows in distinct banks), H <= 4096
  static constexpr int SB_WARP = 32 * (4096 / 64 + 1) * 4;
  static constexpr int OFF_BAR = OFF_SB + (kRouter ? kEpiWarps * SB_WARP : 0);
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // + barriers, alignment slack
};
static_assert(Cfg<MODE_W1>::SMEM_BYTES <= 227 * 1024 && Cfg<MODE_ROUTER>::SMEM_BYTES <= 227 * 1024, "shared memory");

struct Args {
  int T;        // tokens
  int H;        // inputs per token in u
  int KT;       // K steps in all (router: H/64; W1: (H + E)/64)
  int KTu;      // K steps over u (H/64)
  int M;        // output rows (E or P), a multiple of 128
  int m_tiles;  // M / 128
  int n_tiles;  // m_tiles * ceil(T / 64)
  // router
  const uint8_t* rows;  // 8-bit row records: H codes, then H/64 fp16 scales, then H/64 fp16 biases
  int rec;              // bytes per record
  const float* beta;    // [M] or null
  float* logits;        // [T][M]
  // W1
  const int32_t* sel;  // [T][K] executed experts (clamped into [0, E))
  int K;
  int E;
  const uint16_t* b1;  // [M] fp16
  float* z;            // [T][M]
  int* err;
  long long timeout_ns;
};

// A: router codes (uint8 {H, E} over the records, boxes of 128 bytes x 128 rows) or W1 (fp16 {H + E, P}, boxes
// of 64 x 128); u: bf16 {H, T}, boxes of 64 x 64.  All 128-byte swizzled.
struct Maps {
  CUtensorMap a, u;
};

MOE_DEV uint32_t parity(int count, int stages) { return static_cast<uint32_t>(count / stages) & 1u; }

// Instruction descriptor, kind::f16 with bf16 A and B (K-major), fp32 accumulator, M = 128, N = n.
MOE_DEV uint32_t instr_desc_bf16(int n) { return tc::instr_desc(n) | (1u << 7) | (1u << 10); }

MOE_DEV uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Four 8-bit codes (byte i = code of element i) -> bf16 (q - 128) of elements (0, 1) and (2, 3).  A code byte
// placed under the exponent of 2^23 gives 2^23 + q exactly; subtracting 2^23 + 128 leaves q - 128, which bf16
// holds exactly.
MOE_DEV uint2 codes_to_bf16(uint32_t w) {
  constexpr float kOff = 8388736.0f;  // 2^23 + 128
  const float f0 = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650)) - kOff;
  const float f1 = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7651)) - kOff;
  const float f2 = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7652)) - kOff;
  const float f3 = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7653)) - kOff;
  return make_uint2(bf16x2_bits(f0, f1), bf16x2_bits(f2, f3));
}

// Two fp16 values -> their exact split into bf16 hi + lo.
MOE_DEV void split_f16x2(uint32_t w, uint32_t& hi, uint32_t& lo) {
  const float2 f = __half22float2(as_h2(w));
  hi = bf16x2_bits(f.x, f.y);
  const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
  lo = bf16x2_bits(f.x - h0, f.y - h1);
}

// Sum of the 8 bf16 values of a 16-byte chunk added to s, in element order.
MOE_DEV float add_bf16x8(float s, uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s += __uint_as_float(w[i] << 16);
    s += __uint_as_float(w[i] & 0xFFFF0000u);
  }
  return s;
}

template <int MODE>
__global__ void __launch_bounds__(Cfg<MODE>::kThreads, 1) dense_kernel(const __grid_constant__ Maps maps,
                                                                        const __grid_constant__ Args a) {
  using C = Cfg<MODE>;
  constexpr bool kRouter = C::kRouter;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = sm + C::OFF_A;
  uint8_t* smB = sm + C::OFF_B;
  uint8_t* smRaw = sm + C::OFF_RAW;
  float* Us = reinterpret_cast<float*>(sm + C::OFF_U);  // router: [NACC][BN] group sums
  uint8_t* smSB = sm + C::OFF_SB;  // router: per epilogue warp [32][H/64 + 1] words of scale, bias pairs
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + RSTAGES;
  uint64_t* b_full = raw_empty + RSTAGES;
  uint64_t* a_full = b_full + STAGES;
  uint64_t* st_empty = a_full + STAGES;  // both operand stages of a step are free
  uint64_t* acc_full = st_empty + STAGES;
  uint64_t* acc_empty = acc_full + C::NA;
  uint64_t* u_full = acc_empty + C::NA;  // router: the group sums of Us[b] are written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(u_full + C::NA);

  const int KT = a.KT, n_tiles = a.n_tiles;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < RSTAGES; ++s) {
      bar_init(raw_full + s, 1);
      bar_init(raw_empty + s, kCvtWarps);
    }
    for (int s = 0; s < STAGES; ++s) {
      bar_init(b_full + s, 1);
      bar_init(a_full + s, kCvtWarps);
      // router: the converting warps also read the token stage (group sums) before it may be refilled
      bar_init(st_empty + s, kRouter ? 1 + kCvtWarps : C::kMma);
    }
    for (int s = 0; s < C::NA; ++s) {
      bar_init(acc_full + s, kRouter ? 1 : C::kMma);
      bar_init(acc_empty + s, kEpiWarps);
      bar_init(u_full + s, kCvtWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sa(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  int fail = 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int n_raw = 0, gg = 0;
#pragma unroll 1
      for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x) {
        const int y = (ti % a.m_tiles) * BM, t0 = (ti / a.m_tiles) * BN;
#pragma unroll 1
        for (int kt = 0; kt < KT; ++kt, ++gg) {
          if (kt % C::RAW_STEPS == 0) {
            const int rs = n_raw % RSTAGES;
            if (!bar_wait(raw_empty + rs, parity(n_raw, RSTAGES) ^ 1u, a.timeout_ns)) {
              fail = 1;
              break;
            }
            bar_expect_tx(raw_full + rs, RAW_STAGE);
            tma_load_2d(smRaw + rs * RAW_STAGE, &maps.a, kt * BK, y, raw_full + rs);  // bytes or fp16 elements
            ++n_raw;
          }
          const int s = gg % STAGES;
          if (!bar_wait(st_empty + s, parity(gg, STAGES) ^ 1u, a.timeout_ns)) {
            fail = 1;
            break;
          }
          if (kt < a.KTu) {
            bar_expect_tx(b_full + s, B_STAGE);
            tma_load_2d(smB + s * B_STAGE, &maps.u, kt * BK, t0, b_full + s);
          } else {
            bar_arrive(b_full + s);  // multi-hot step: the converting warps write the token stage
          }
        }
      }
      if (fail) {  // let the copies already issued land before the CTA can leave
#pragma unroll 1
        for (int q = n_raw > RSTAGES ? n_raw - RSTAGES : 0; q < n_raw; ++q)
          bar_wait(raw_full + q % RSTAGES, parity(q, RSTAGES), a.timeout_ns);
#pragma unroll 1
        for (int q = gg > STAGES ? gg - STAGES : 0; q < gg; ++q)
          bar_wait(b_full + q % STAGES, parity(q, STAGES), a.timeout_ns);
      }
    }
  } else if (warp < C::kWarpCvt0) {
    // ---------------------------------------------------------------- MMA issue
    const int mw = warp - 1;
    if (lane == 0) {
      const uint32_t idesc = instr_desc_bf16(BN);
      int gg = 0, it = 0, last = -1;
      uint32_t last_par = 0;
#pragma unroll 1
      for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x, ++it) {
        const int ab = it & 1;
        if (!kRouter) {
          if (!bar_wait(acc_empty + ab, parity(it, 2) ^ 1u, a.timeout_ns)) {
            fail = 1;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        }
#pragma unroll 1
        for (int kt = 0; kt < KT; ++kt, ++gg) {
          const int s = gg % STAGES;
          if (kRouter) {
            const int b = gg % NACC;  // issued by MMA warp b % kMma
            if (b % C::kMma != mw) continue;
            if (!bar_wait(acc_empty + b, parity(gg, NACC) ^ 1u, a.timeout_ns)) {
              fail = 1;
              break;
            }
          }
          if (!bar_wait(a_full + s, parity(gg, STAGES), a.timeout_ns) ||
              !bar_wait(b_full + s, parity(gg, STAGES), a.timeout_ns)) {
            fail = 1;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t a0 = sa(smA + s * C::A_STAGE), b0 = sa(smB + s * B_STAGE);
          if (kRouter) {
            const int b = gg % NACC;
            const uint32_t d = tmem + static_cast<uint32_t>(b * BN);
#pragma unroll
            for (int c = 0; c < 4; ++c) mma_f16(d, smem_desc(a0 + c * 32), smem_desc(b0 + c * 32), idesc, c != 0);
            mma_commit(st_empty + s);
            mma_commit(acc_full + b);
            last = b;
            last_par = parity(gg, NACC);
          } else {
            const uint32_t d = tmem + static_cast<uint32_t>(ab * 4 * BN);
#pragma unroll
            for (int c = mw; c < 4; c += C::kMma) {
              mma_f16(d + c * BN, smem_desc(a0 + c * 32), smem_desc(b0 + c * 32), idesc, kt != 0);
              mma_f16(d + c * BN, smem_desc(a0 + A_SUB + c * 32), smem_desc(b0 + c * 32), idesc, 1);
            }
            mma_commit(st_empty + s);
          }
        }
        if (!kRouter) {
          mma_commit(acc_full + ab);  // also on failure: completes once the MMAs issued into it are done
          last = ab;
          last_par = parity(it, 2);
        }
      }
      // never release TMEM with MMAs in flight
      if (fail && last >= 0) bar_wait(acc_full + last, last_par, a.timeout_ns);
    }
  } else if (warp < C::kWarpEpi0) {
    // ---------------------------------------------------------------- converting warps
    const int d = tid - 32 * C::kWarpCvt0;  // 0..255
    // lanes l and l+8 take the two halves of one row; a 128-byte wavefront covers 8 consecutive rows
    const int r = 16 * (d >> 5) + (lane & 7) + 8 * (lane >> 4), h = (lane >> 3) & 1;
    const int tt = d >> 2, qq = d & 3;  // router group sums: token row tt, quarter qq of its 64 values
    int gg = 0, nr = 0;
#pragma unroll 1
    for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x) {
      const int t0 = (ti / a.m_tiles) * BN;
#pragma unroll 1
      for (int kt = 0; kt < KT; ++kt, ++gg) {
        const int rs = nr % RSTAGES, j = kt % C::RAW_STEPS;
        if (__any_sync(0xffffffffu, j == 0 && !bar_wait(raw_full + rs, parity(nr, RSTAGES), a.timeout_ns))) {
          fail = 1;
          break;
        }
        // 16-byte chunk c of row r sits at c ^ (r % 8) under the 128-byte swizzle
        const uint8_t* rrow = smRaw + rs * RAW_STAGE + r * 128;
        uint4 q[4];
        if (kRouter) {  // 32 codes: chunks 4j + 2h and 4j + 2h + 1
          q[0] = *reinterpret_cast<const uint4*>(rrow + (((4 * j + 2 * h) ^ (r & 7)) << 4));
          q[1] = *reinterpret_cast<const uint4*>(rrow + (((4 * j + 2 * h + 1) ^ (r & 7)) << 4));
        } else {  // 32 fp16: chunks 4h .. 4h + 3
#pragma unroll
          for (int i = 0; i < 4; ++i) q[i] = *reinterpret_cast<const uint4*>(rrow + (((4 * h + i) ^ (r & 7)) << 4));
        }
        if (j == C::RAW_STEPS - 1 || kt == KT - 1) {
          __syncwarp();
          if (lane == 0) bar_arrive(raw_empty + rs);
          ++nr;
        }
        uint4 o[4], lo[4];
        if (kRouter) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint2 c0 = codes_to_bf16(q[i].x), c1 = codes_to_bf16(q[i].y);
            const uint2 c2 = codes_to_bf16(q[i].z), c3 = codes_to_bf16(q[i].w);
            o[2 * i] = make_uint4(c0.x, c0.y, c1.x, c1.y);
            o[2 * i + 1] = make_uint4(c2.x, c2.y, c3.x, c3.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            split_f16x2(q[i].x, o[i].x, lo[i].x);
            split_f16x2(q[i].y, o[i].y, lo[i].y);
            split_f16x2(q[i].z, o[i].z, lo[i].z);
            split_f16x2(q[i].w, o[i].w, lo[i].w);
          }
        }
        const int s = gg % STAGES;
        if (__any_sync(0xffffffffu, !bar_wait(st_empty + s, parity(gg, STAGES) ^ 1u, a.timeout_ns))) {
          fail = 1;  // the MMA may still read this stage
          break;
        }
        uint8_t* dd = smA + s * C::A_STAGE + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          *reinterpret_cast<uint4*>(dd + (((4 * h + i) ^ (r & 7)) << 4)) = o[i];
          if (!kRouter) *reinterpret_cast<uint4*>(dd + A_SUB + (((4 * h + i) ^ (r & 7)) << 4)) = lo[i];
        }
        if (!kRouter && kt >= a.KTu) {
          // multi-hot token rows: element e0 + k of token t = how many of its K selections are e0 + k
          const int e0 = (kt - a.KTu) * BK;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int idx = 2 * d + i, trow = idx >> 3, c = idx & 7, t = t0 + trow;
            float cnt[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (t < a.T) {
              for (int k = 0; k < a.K; ++k) {
                int e = a.sel[static_cast<size_t>(t) * a.K + k];
                e = e < 0 ? 0 : (e >= a.E ? a.E - 1 : e);
                const int rel = e - e0 - 8 * c;
#pragma unroll
                for (int m = 0; m < 8; ++m) cnt[m] += rel == m ? 1.f : 0.f;
              }
            }
            const uint4 v = make_uint4(bf16x2_bits(cnt[0], cnt[1]), bf16x2_bits(cnt[2], cnt[3]),
                                       bf16x2_bits(cnt[4], cnt[5]), bf16x2_bits(cnt[6], cnt[7]));
            *reinterpret_cast<uint4*>(smB + s * B_STAGE + trow * 128 + ((c ^ (trow & 7)) << 4)) = v;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(a_full + s);
        if (kRouter) {
          // group sum of token row tt: four lanes take 16 values each, in element order, then add pairwise
          if (__any_sync(0xffffffffu, !bar_wait(b_full + s, parity(gg, STAGES), a.timeout_ns))) {
            fail = 1;
            break;
          }
          const uint8_t* brow = smB + s * B_STAGE + tt * 128;
          const uint4 v0 = *reinterpret_cast<const uint4*>(brow + (((2 * qq) ^ (tt & 7)) << 4));
          const uint4 v1 = *reinterpret_cast<const uint4*>(brow + (((2 * qq + 1) ^ (tt & 7)) << 4));
          __syncwarp();
          if (lane == 0) bar_arrive(st_empty + s);  // this warp's reads of the token stage are done
          float sum = add_bf16x8(add_bf16x8(0.f, v0), v1);
          sum += __shfl_xor_sync(0xffffffffu, sum, 1);
          sum += __shfl_xor_sync(0xffffffffu, sum, 2);
          const int b = gg % NACC;
          if (__any_sync(0xffffffffu, !bar_wait(acc_empty + b, parity(gg, NACC) ^ 1u, a.timeout_ns))) {
            fail = 1;  // the epilogue may still read Us[b]
            break;
          }
          if (qq == 0) Us[b * BN + tt] = sum;
          __syncwarp();
          if (lane == 0) bar_arrive(u_full + b);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (TMEM lane quadrant = warp % 4)
    const int ew = warp - C::kWarpEpi0;
    const int quad = warp & 3;
    const int c0 = 32 * (ew >> 2);  // token columns [c0, c0 + 32)
    const int L = quad * 32 + lane;  // TMEM lane = tile row
    const uint32_t lane_off = (static_cast<uint32_t>(quad) * 32u) << 16;
    int gg = 0, it = 0;
#pragma unroll 1
    for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x, ++it) {
      const int row = (ti % a.m_tiles) * BM + L, t0 = (ti / a.m_tiles) * BN;
      float v[32];
      if (kRouter) {
        // this warp's 32 rows' scale and bias runs (H/64 words per row: H/64 fp16 scales, then H/64 fp16
        // biases) into its own shared-memory copy: one coalesced row per step, no cross-warp dependence
        const int SW = KT, SBW = KT + 1;
        uint32_t* sbs = reinterpret_cast<uint32_t*>(smSB + ew * C::SB_WARP);
        const uint8_t* sb0 = a.rows + static_cast<size_t>(row - lane) * a.rec + a.H;
#pragma unroll 1
        for (int w0 = 0; w0 < SW; w0 += 32) {  // 32 independent loads in flight, then the stores
          const int wd = w0 + lane;
          uint32_t tmp[32];
#pragma unroll
          for (int rr = 0; rr < 32; ++rr)
            tmp[rr] = wd < SW ? reinterpret_cast<const uint32_t*>(sb0 + static_cast<size_t>(rr) * a.rec)[wd] : 0u;
#pragma unroll
          for (int rr = 0; rr < 32; ++rr)
            if (wd < SW) sbs[rr * SBW + wd] = tmp[rr];
        }
        __syncwarp();
        const uint16_t* sbr = reinterpret_cast<const uint16_t*>(sbs + lane * SBW);  // scales, then biases
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
#pragma unroll 1
        for (int kt = 0; kt < KT; ++kt, ++gg) {
          const int b = gg % NACC;
          const float s = half_bits_to_float(sbr[kt]);
          const float bp = fmaf(128.f, s, half_bits_to_float(sbr[KT + kt]));  // b + 128 s, one rounding
          if (__any_sync(0xffffffffu, !bar_wait(acc_full + b, parity(gg, NACC), a.timeout_ns) ||
                                          !bar_wait(u_full + b, parity(gg, NACC), a.timeout_ns))) {
            fail = 1;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          float D[32];
          tmem_ld32(tmem + static_cast<uint32_t>(b * BN + c0) + lane_off, D);
          float U[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 u4 = reinterpret_cast<const float4*>(Us + b * BN + c0)[j];
            U[4 * j] = u4.x;
            U[4 * j + 1] = u4.y;
            U[4 * j + 2] = u4.z;
            U[4 * j + 3] = u4.w;
          }
          asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
          __syncwarp();
          if (lane == 0) bar_arrive(acc_empty + b);  // accumulator and group sums read
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v[j] = fmaf(s, D[j], v[j]);
            v[j] = fmaf(bp, U[j], v[j]);
          }
        }
        __syncwarp();  // the next tile's scales overwrite these
        if (fail) break;
        const float beta = a.beta ? a.beta[row] : 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = t0 + c0 + j;
          if (t < a.T) a.logits[static_cast<size_t>(t) * a.M + row] = v[j] + beta;
        }
      } else {
        const int ab = it & 1;
        const float bias = half_bits_to_float(a.b1[row]);
        if (__any_sync(0xffffffffu, !bar_wait(acc_full + ab, parity(it, 2), a.timeout_ns))) {
          fail = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t taddr = tmem + static_cast<uint32_t>(ab * 4 * BN + c0) + lane_off;
        tmem_ld32(taddr, v);
#pragma unroll 1
        for (int ch = 1; ch < 4; ++ch) {
          float w[32];
          tmem_ld32(taddr + ch * BN, w);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] += w[j];
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) bar_arrive(acc_empty + ab);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = t0 + c0 + j;
          if (t < a.T) a.z[static_cast<size_t>(t) * a.M + row] = silu(v[j] + bias);
        }
      }
    }
  }
  if (fail) report(a.err, 5);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
}

}  // namespace dense
}  // namespace moe
