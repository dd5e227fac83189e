// Grouped GEMM on the 5th-generation tensor cores (tcgen05) for many-token
// batches: persistent, warp-specialised, int4 weight stream by TMA.
//
// Per expert bucket D[o][t] = sum_k W[o][k] * X[t][k] ("swap AB": 128 weight
// rows are the MMA M side, the bucket's tokens the N side).  A tile is 128
// weight rows x up to 128 tokens (the MMA's N is the tile's token count rounded
// up to 16); K advances one quantisation group (64) per step, four steps per
// pass.  One CTA per SM walks the device-built tile list (tiles c, c + grid,
// ...), and every role runs the same sequence of (tile, pass, step), so the
// pipeline stays full across tiles:
//  * warp 0, one lane (weight TMA, running ahead as far as its buffers allow):
//    per tile the fp16 scales and biases of its 128 rows (a box of a 3-D byte
//    map {record bytes, rows, experts} over the expert pool, two buffers when
//    they fit); per pass the 128 code bytes of each row (a box of a second map
//    over the same bytes, 128-byte swizzle, 16 KB, three stages);
//  * warp 2, one lane (token TMA): per step the step's token rows (2-D map,
//    128-byte swizzle, boxes of 32 rows, only as many as the tile has tokens;
//    four 16 KB stages);
//  * warp 1, one lane (MMA): per step four tcgen05.mma kind::f16 (one per 16-wide
//    K slice) in straight-line code -- A from tensor memory, B (tokens) from
//    shared memory -- into the tile's accumulator (two 128-column TMEM
//    accumulators, tiles alternate); one thread issues the whole tile: a
//    predicate, a loop or a wait around an MMA costs the issuing thread more
//    than the MMA's own tensor-core time, so work per instruction (N up to 128)
//    and few instructions around it are what count;
//  * 8 warps dequantise a pass (one raw stage, four K steps) at a time straight
//    into tensor memory (two passes in flight): a warp owns the TMEM lanes of
//    its quadrant (warp % 4), thread = weight row, the quadrant's two warps the
//    two halves of a step's 64 inputs; a thread reads 16 code bytes per step
//    (conflict-free under the swizzle), forms w = q*s + b in fp16 (one rounding)
//    and stores 16 columns with tcgen05.st; one mbarrier hand-off per pass in
//    each direction.  K inside each 8-element block is in "pair order" (q_j,
//    q_{j+4}), the order the magic-exponent unpacking produces; the token operand
//    is stored in the same order, so the products are those of the plain order;
//  * 8 epilogue warps (TMEM lane quadrant = warp % 4, two warps per quadrant,
//    64 token columns each in two blocks of 32): drain the finished accumulator
//    with tcgen05.ld while the next tile's main loop runs: SwiGLU of interleaved
//    gate/up rows (output in pair order, the next GEMM's token operand) or the
//    down projection's LoRA delta and gating weight; staged in shared memory for
//    coalesced fp16 stores; then the accumulator is released.
// Every wait is bounded: a role whose wait runs out stops issuing copies or
// MMAs and records MOE_ERR_TIMEOUT; before the CTA leaves, the copies, MMAs and
// tensor-memory stores it issued are waited for (bounded).
#pragma once

#include "tc_primitives.cuh"

namespace moe {
namespace gg3 {

using tc::bar_arrive;
using tc::bar_expect_tx;
using tc::bar_init;
using tc::bar_test;
using tc::bar_wait;
using tc::EPI_DOWN;
using tc::EPI_SWIGLU;
using tc::instr_desc;
using tc::mma_commit;
using tc::mma_f16_ts;
using tc::sa;
using tc::smem_desc;
using tc::tma_load_2d;
using tc::tmem_ld16;
using tc::tmem_ld32;
using tc::tmem_st16;
using tc::tmem_st_wait;
using tc::Tile;

constexpr int BM = 128;
constexpr int BN = 128;     // tokens per tile
constexpr int BK = 64;
constexpr int BROWS = 32;   // token rows per TMA box
constexpr int RGROUPS = 4;  // K steps per pass = quantisation groups per raw code load: 128-byte TMA rows
                            // (narrower rows cap the TMA request rate well below the HBM bandwidth)
constexpr int RSTAGES = 3;  // raw code stages (16 KB each): the weight bytes in flight per SM
constexpr int BSTAGES = 4;  // token stages (16 KB each)
constexpr int APASS = 2;    // dequantised weight passes in tensor memory (RGROUPS stages of 32 columns each)
constexpr int kDqWarps = 8;
constexpr int kDq = 32 * kDqWarps;
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant, splitting the tile's token columns
constexpr int kEpi = 32 * kEpiWarps;
constexpr int kThreads = 96 + kDq + kEpi;  // weight TMA warp, MMA warp, token TMA warp, dequant, epilogue warps
constexpr int kWarpDq0 = 3;                // first dequantising warp
constexpr int kWarpEpi0 = kWarpDq0 + kDqWarps;
constexpr int RAW_STAGE = BM * 32 * RGROUPS;
constexpr int B_STAGE = BN * BK * 2;
constexpr int A_COLS = BK / 2;    // TMEM columns of one dequantised weight stage (two fp16 per column)
constexpr int ACC_COLS = 2 * BN;  // TMEM: two tiles' accumulators, then the weight stages
constexpr uint32_t TMEM_COLS = 512;
constexpr int STAGE_OUT = BN * BM * 2;  // epilogue staging: up to BN tokens x 128 fp16
constexpr int OFF_B = 0;
constexpr int OFF_RAW = OFF_B + BSTAGES * B_STAGE;
constexpr int LORA_T = 2 * BN * 32 * 4;  // epilogue staging of the tile's LoRA t vectors (two sets, r <= 32) ...
constexpr int OFF_OUT = OFF_RAW + RSTAGES * RAW_STAGE;
constexpr int OFF_LT = OFF_OUT + STAGE_OUT;
constexpr int OFF_RS = OFF_LT + LORA_T;  // ... of its gating weights ...
static_assert(BN * BM * 2 <= LORA_T, "a tile of precomputed fp16 deltas fits the LoRA staging area");
constexpr int LORA_B = BM * 32 * 4;
constexpr int OFF_BL = OFF_RS + BN * 4;  // ... and of its rows' LoRA B values times the LoRA scale, [i][row]
constexpr int OFF_SB = OFF_BL + LORA_B;
static_assert(ACC_COLS + APASS * RGROUPS * A_COLS <= static_cast<int>(TMEM_COLS) && BK == 64 && kDqWarps == 8,
              "tensor memory plan");

// Bytes per row of the scale/bias box: the K/64 scales and K/64 biases (4*K/64 bytes), at least one 16-byte
// TMA unit (the row record's zero padding covers the rest).
__host__ __device__ constexpr int sb_row_bytes(int K) { return (4 * (K / 64) + 15) / 16 * 16; }
// Dynamic shared memory for reduction length K with nsb scale/bias buffers (+ barriers, alignment slack).
__host__ __device__ constexpr int smem_bytes(int K, int nsb) { return OFF_SB + nsb * BM * sb_row_bytes(K) + 512 + 1024; }
// Scale/bias buffers for reduction length K: two (the next tile's scales load during this tile) when they fit.
__host__ __device__ constexpr int sb_buffers(int K) { return smem_bytes(K, 2) <= 227 * 1024 ? 2 : 1; }

struct Args {
  const Tile* tiles;
  const int* n_tiles;
  int E;
  int K;
  int epi;
  uint16_t* out;
  int out_ld;
  const float* row_scale;
  const float* lora_t1;  // routed adapters' t vectors [row][r] (SwiGLU: the gate's; down: the down's)
  const float* lora_t2;  // SwiGLU: the up projection's
  const uint16_t* lora_Bex;
  const uint16_t* lora_Bgu_ex;  // SwiGLU, routed: per-expert B [E][2I][r] in the block's interleaved row order
  // the shared expert's unmerged LoRA deltas, computed per token beforehand: fp16 [token][lora_D_ld] (output
  // rows in the weight matrix's order); shared rows start at tile row lora_D_row0 (null: none)
  const uint16_t* lora_D;
  int lora_D_ld;
  int lora_D_row0;
  int lora_r;
  float lora_scale;
  int* err;
  long long timeout_ns;
  int drop_tile;  // test hook: the CTA working on this tile never marks its first weight stage full (-1: off)
  int nsb;        // scale/bias buffers (sb_buffers(K))
};

// 3-D byte maps {record bytes, rows, experts} over the weight matrix of every expert block (pool) and of the
// shared expert's block (one expert): boxes of the 128 code bytes of four groups x 128 rows (128-byte swizzle),
// and of the scale/bias bytes x 128 rows.  2-D fp16 map of the token operand [rows][K], boxes of 64 x 32,
// 128-byte swizzle.
struct Maps {
  CUtensorMap pool_codes, pool_sb, shared_codes, shared_sb, tokens;
};

MOE_DEV void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(sa(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(sa(bar))
      : "memory");
}

// One int4 word -> 8 fp16 weights q*s + b in pair order ((w_j, w_{j+4}) for j = 0..3).  The codes come out of
// the magic-exponent unpacking exactly (lo nibbles: (1024 + q) - 1024; hi nibbles: (1024 + 16 q) / 16 - 64).
MOE_DEV uint4 dequant_pair_order(uint32_t w, __half2 s2, __half2 b2) {
  const uint32_t kMagic = 0x64006400u;
  const uint32_t lo0 = lop_and_or(w, 0x000F000Fu, kMagic);
  const uint32_t hi0 = lop_and_or(w, 0x00F000F0u, kMagic);
  const uint32_t w8 = w >> 8;
  const uint32_t lo1 = lop_and_or(w8, 0x000F000Fu, kMagic);
  const uint32_t hi1 = lop_and_or(w8, 0x00F000F0u, kMagic);
  const __half2 k1024 = __half2half2(__ushort_as_half(0x6400));  // 1024
  const __half2 k16th = __half2half2(__ushort_as_half(0x2C00));  // 1/16
  const __half2 km64 = __half2half2(__ushort_as_half(0xD400));   // -64
  const __half2 q0 = __hsub2(as_h2(lo0), k1024), q1 = __hfma2(as_h2(hi0), k16th, km64);
  const __half2 q2 = __hsub2(as_h2(lo1), k1024), q3 = __hfma2(as_h2(hi1), k16th, km64);
  return make_uint4(h2_bits(__hfma2(q0, s2, b2)), h2_bits(__hfma2(q1, s2, b2)), h2_bits(__hfma2(q2, s2, b2)),
                    h2_bits(__hfma2(q3, s2, b2)));
}

MOE_DEV uint32_t parity(int count, int stages) { return static_cast<uint32_t>(count / stages) & 1u; }

// Barrier of the 256 epilogue threads (named barrier 1).  The warp is reconverged first and the barrier is the
// non-aligned form: the lanes of a warp may come from loops of different trip counts, and the aligned form
// would let a warp that arrives diverged release the others early.
MOE_DEV void epi_sync() {
  __syncwarp();
  asm volatile("barrier.sync 1, 256;" ::: "memory");
}

// OR of v over the 256 epilogue threads (named barrier 1), so that they take the same branch.
MOE_DEV bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.cta.red.or.pred q, 1, 256, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1) grouped_gemm3_kernel(const __grid_constant__ Maps maps,
                                                                    const __grid_constant__ Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int KT = a.K / BK;
  const int SB_ROW = sb_row_bytes(a.K);  // scales at byte 0, biases at byte 2*KT of a row
  uint8_t* smB = sm + OFF_B;
  uint8_t* smRaw = sm + OFF_RAW;
  uint16_t* stage = reinterpret_cast<uint16_t*>(sm + OFF_OUT);
  uint8_t* smSB = sm + OFF_SB;  // nsb buffers of BM * SB_ROW bytes
  const int nsb = a.nsb;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smSB + nsb * BM * SB_ROW);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + RSTAGES;
  uint64_t* b_full = raw_empty + RSTAGES;
  uint64_t* b_empty = b_full + BSTAGES;
  uint64_t* a_full = b_empty + BSTAGES;   // [APASS] a pass's weight stages are in tensor memory
  uint64_t* a_empty = a_full + APASS;     // [APASS] the MMA is done with a pass's weight stages
  uint64_t* sb_full = a_empty + APASS;    // [2]
  uint64_t* sb_empty = sb_full + 2;       // [2]
  uint64_t* acc_full = sb_empty + 2;      // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int n_tiles = *a.n_tiles;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < RSTAGES; ++s) {
      bar_init(raw_full + s, 1);
      bar_init(raw_empty + s, kDqWarps);  // one elected arrival per warp
    }
    for (int s = 0; s < BSTAGES; ++s) {
      bar_init(b_full + s, 1);
      bar_init(b_empty + s, 1);
    }
    for (int s = 0; s < APASS; ++s) {
      bar_init(a_full + s, kDqWarps);
      bar_init(a_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      bar_init(sb_full + s, 1);
      bar_init(sb_empty + s, kDqWarps);
      bar_init(acc_full + s, 1);
      bar_init(acc_empty + s, kEpiWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // the MMA warp owns the TMEM allocation
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sa(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  int fail = 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- weight TMA producer: scales, raw codes
    // (runs ahead of the token copies as far as its buffers allow)
    if (lane == 0) {
      int n_raw = 0, n_sb = 0;  // copies issued so far (stage counters)
#pragma unroll 1
      for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x) {
        const Tile tile = a.tiles[ti];
        const bool sh = tile.e >= a.E;
        const CUtensorMap* cmap = sh ? &maps.shared_codes : &maps.pool_codes;
        const CUtensorMap* smap = sh ? &maps.shared_sb : &maps.pool_sb;
        const int ez = sh ? 0 : tile.e, y = tile.mt * BM;
        const int tb = n_sb % nsb;
        if (!bar_wait(sb_empty + tb, parity(n_sb, nsb) ^ 1u, a.timeout_ns)) {
          fail = 1;
          break;
        }
        bar_expect_tx(sb_full + tb, static_cast<uint32_t>(BM * SB_ROW));
        tma_load_3d(smSB + tb * BM * SB_ROW, smap, a.K / 2, y, ez, sb_full + tb);
        ++n_sb;
#pragma unroll 1
        for (int kt = 0; kt < KT; kt += RGROUPS) {
          const int rs = n_raw % RSTAGES;
          if (!bar_wait(raw_empty + rs, parity(n_raw, RSTAGES) ^ 1u, a.timeout_ns)) {
            fail = 1;
            break;
          }
          bar_expect_tx(raw_full + rs, RAW_STAGE);
          tma_load_3d(smRaw + rs * RAW_STAGE, cmap, kt * 32, y, ez, raw_full + rs);
          ++n_raw;
        }
      }
      if (fail) {  // let the copies already issued land before the CTA can leave
#pragma unroll 1
        for (int q = n_raw > RSTAGES ? n_raw - RSTAGES : 0; q < n_raw; ++q)
          bar_wait(raw_full + q % RSTAGES, parity(q, RSTAGES), a.timeout_ns);
#pragma unroll 1
        for (int q = n_sb > nsb ? n_sb - nsb : 0; q < n_sb; ++q) bar_wait(sb_full + q % nsb, parity(q, nsb), a.timeout_ns);
      }
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- token TMA producer
    if (lane == 0) {
      int n_b = 0;
#pragma unroll 1
      for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x) {
        const Tile tile = a.tiles[ti];
        const int nb = (tile.n + BROWS - 1) / BROWS;
#pragma unroll 1
        for (int kt = 0; kt < KT; ++kt) {
          const int bs = n_b % BSTAGES;
          if (!bar_wait(b_empty + bs, parity(n_b, BSTAGES) ^ 1u, a.timeout_ns)) {
            fail = 1;
            break;
          }
          bar_expect_tx(b_full + bs, static_cast<uint32_t>(nb * BROWS * BK * 2));
#pragma unroll 1
          for (int i = 0; i < nb; ++i)
            tma_load_2d(smB + bs * B_STAGE + i * BROWS * BK * 2, &maps.tokens, kt * BK, tile.row0 + i * BROWS,
                        b_full + bs);
          ++n_b;
        }
      }
      if (fail) {
#pragma unroll 1
        for (int q = n_b > BSTAGES ? n_b - BSTAGES : 0; q < n_b; ++q)
          bar_wait(b_full + q % BSTAGES, parity(q, BSTAGES), a.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      int n_b = 0, np = 0, it = 0, last_ab = -1;
      uint32_t last_par = 0;
#pragma unroll 1
      for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x, ++it) {
        const Tile tile = a.tiles[ti];
        const int ab = it & 1;
        if (!bar_wait(acc_empty + ab, parity(it, 2) ^ 1u, a.timeout_ns)) {
          fail = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t d = tmem + static_cast<uint32_t>(ab * BN);
        const uint32_t idesc = instr_desc((tile.n + 15) & ~15);
#pragma unroll 1
        for (int kt = 0; kt < KT && !fail; kt += RGROUPS, ++np) {
          const int ps = np % APASS, nst = KT - kt < RGROUPS ? KT - kt : RGROUPS;
          if (!bar_wait(a_full + ps, parity(np, APASS), a.timeout_ns)) {
            fail = 1;
            break;
          }
#pragma unroll 1
          for (int st = 0; st < nst; ++st, ++n_b) {
            const int bs = n_b % BSTAGES;
            if (!bar_wait(b_full + bs, parity(n_b, BSTAGES), a.timeout_ns)) {
              fail = 1;
              break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            // the step's four 16-wide K slices: A 8 TMEM columns each, B 32 bytes each (the descriptor's
            // start-address field moves by 2)
            const uint32_t a0 = tmem + static_cast<uint32_t>(ACC_COLS + (ps * RGROUPS + st) * A_COLS);
            const uint64_t b0 = smem_desc(sa(smB + bs * B_STAGE));
            mma_f16_ts(d, a0, b0, idesc, (kt | st) != 0);
            mma_f16_ts(d, a0 + 8, b0 + 2, idesc, 1u);
            mma_f16_ts(d, a0 + 16, b0 + 4, idesc, 1u);
            mma_f16_ts(d, a0 + 24, b0 + 6, idesc, 1u);
            mma_commit(b_empty + bs);
          }
          mma_commit(a_empty + ps);
        }
        mma_commit(acc_full + ab);  // also on failure: completes once every MMA issued into this buffer has
        last_ab = ab;
        last_par = parity(it, 2);
      }
      // never release TMEM with MMAs in flight: wait for the last commit
      if (fail && last_ab >= 0) bar_wait(acc_full + last_ab, last_par, a.timeout_ns);
    }
  } else if (warp < kWarpEpi0) {
    // ---------------------------------------------------------------- dequantising warps
    const int d = tid - 32 * kWarpDq0;
    // a warp writes the TMEM lanes of its quadrant (warp % 4): thread = weight row r, and the two warps of a
    // quadrant take the two halves h of each step's 64 inputs
    const int quad = warp & 3, h = (warp - kWarpDq0) >> 2, r = 32 * quad + lane;
    const uint32_t a_lane = tmem + (static_cast<uint32_t>(32 * quad) << 16) + ACC_COLS + 16 * h;
    const bool vec8 = (KT & 7) == 0;
    int np = 0, it = 0;
#pragma unroll 1
    for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x, ++it) {
      const int tb = it % nsb;
      const uint16_t* sbr = reinterpret_cast<const uint16_t*>(smSB + tb * BM * SB_ROW + r * SB_ROW);
      if (__any_sync(0xffffffffu, !bar_wait(sb_full + tb, parity(it, nsb), a.timeout_ns))) {
        fail = 1;
        break;
      }
      // a row's scale/bias run sits in one bank for all rows: read them 8 groups at a time
      uint4 s8 = make_uint4(0, 0, 0, 0), b8 = s8;
#pragma unroll 1
      for (int kt = 0; kt < KT; kt += RGROUPS, ++np) {  // one raw stage (RGROUPS steps) per pass
        const int nst = KT - kt < RGROUPS ? KT - kt : RGROUPS;
        if (vec8 && (kt & 7) == 0) {
          s8 = reinterpret_cast<const uint4*>(sbr)[kt >> 3];
          b8 = reinterpret_cast<const uint4*>(sbr + KT)[kt >> 3];
        }
        uint32_t sw[2], bw[2];  // fp16 pairs: steps (kt, kt + 1), (kt + 2, kt + 3)
        if (vec8) {
          const bool hi = (kt & 7) != 0;
          sw[0] = hi ? s8.z : s8.x;
          sw[1] = hi ? s8.w : s8.y;
          bw[0] = hi ? b8.z : b8.x;
          bw[1] = hi ? b8.w : b8.y;
        } else {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int k0 = kt + 2 * j < KT ? kt + 2 * j : KT - 1, k1 = kt + 2 * j + 1 < KT ? kt + 2 * j + 1 : KT - 1;
            sw[j] = sbr[k0] | (static_cast<uint32_t>(sbr[k1]) << 16);
            bw[j] = sbr[KT + k0] | (static_cast<uint32_t>(sbr[KT + k1]) << 16);
          }
        }
        const int rs = np % RSTAGES;  // raw stages go round once per pass, as the passes do
        if (__any_sync(0xffffffffu, !bar_wait(raw_full + rs, parity(np, RSTAGES), a.timeout_ns))) {
          fail = 1;
          break;
        }
        // chunk (2 st + h) of row r, 128-byte swizzle: 16-byte chunk c of a row sits at c ^ (r % 8)
        const uint8_t* rrow = smRaw + rs * RAW_STAGE + r * 128;
        uint4 q[RGROUPS];
#pragma unroll
        for (int st = 0; st < RGROUPS; ++st)
          q[st] = st < nst ? *reinterpret_cast<const uint4*>(rrow + (((2 * st + h) ^ (r & 7)) << 4))
                           : make_uint4(0, 0, 0, 0);
        __syncwarp();
        if (lane == 0) bar_arrive(raw_empty + rs);
        const int ps = np % APASS;
        if (__any_sync(0xffffffffu, !bar_wait(a_empty + ps, parity(np, APASS) ^ 1u, a.timeout_ns))) {
          fail = 1;  // the MMA may still read this pass's stages
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
        for (int st = 0; st < RGROUPS; ++st) {
          if (st < nst) {
            const uint32_t sp = (st & 1) ? sw[st >> 1] >> 16 : sw[st >> 1] & 0xFFFFu;
            const uint32_t bp = (st & 1) ? bw[st >> 1] >> 16 : bw[st >> 1] & 0xFFFFu;
            const __half2 s2 = __half2half2(__ushort_as_half(static_cast<uint16_t>(sp)));
            const __half2 b2 = __half2half2(__ushort_as_half(static_cast<uint16_t>(bp)));
            const uint4 w0 = dequant_pair_order(q[st].x, s2, b2), w1 = dequant_pair_order(q[st].y, s2, b2);
            const uint4 w2 = dequant_pair_order(q[st].z, s2, b2), w3 = dequant_pair_order(q[st].w, s2, b2);
            const uint32_t v[16] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w,
                                    w2.x, w2.y, w2.z, w2.w, w3.x, w3.y, w3.z, w3.w};
            // inputs 32 h .. 32 h + 31 of the step: columns 16 h .. 16 h + 15 of its stage
            tmem_st16(a_lane + (ps * RGROUPS + st) * A_COLS, v);
          }
        }
        tmem_st_wait();
        // the pass's stages are in tensor memory: hand them to the MMA
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0 && !(kt == 0 && d == 0 && ti == a.drop_tile)) bar_arrive(a_full + ps);
      }
      if (fail) break;
      __syncwarp();
      if (lane == 0) bar_arrive(sb_empty + tb);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (TMEM lane quadrant = warp % 4)
    const int ew = warp - kWarpEpi0;  // 0..7
    const int quad = warp & 3;
    const int chalf = ew >> 2;             // token columns [64 chalf, 64 chalf + 64), two blocks of 32
    const int L = quad * 32 + lane;        // TMEM lane = tile row
    const int et = tid - 32 * kWarpEpi0;  // 0..255 among the epilogue threads
    const int r = a.lora_r;
    float* lt = reinterpret_cast<float*>(sm + OFF_LT);   // [token][r] LoRA t vectors of the tile (two sets)
    float* rsc = reinterpret_cast<float*>(sm + OFF_RS);  // [token] gating weights of the tile
    float* bls = reinterpret_cast<float*>(sm + OFF_BL);  // [i][row] LoRA B of the tile's rows, times the scale
    int it = 0;
#pragma unroll 1
    for (int ti = blockIdx.x; ti < n_tiles && !fail; ti += gridDim.x, ++it) {
      const Tile tile = a.tiles[ti];
      const int ab = it & 1;
      // per-tile inputs of the epilogue, staged once while the accumulator is still being written
      const bool swiglu = a.epi == EPI_SWIGLU;
      const bool up = swiglu && (L & 1) != 0;
      // a routed expert's adapter B rows (SwiGLU: [E][2I][r] in the interleaved row order, out_ld = I; down:
      // [E][H][r]); the shared expert's rows take precomputed deltas instead
      const uint16_t* Bsrc =
          tile.e >= a.E ? nullptr
          : swiglu      ? (a.lora_Bgu_ex ? a.lora_Bgu_ex + static_cast<size_t>(tile.e) * 2 * a.out_ld * r : nullptr)
                        : (a.lora_Bex ? a.lora_Bex + static_cast<size_t>(tile.e) * a.out_ld * r : nullptr);
      const bool dtile = tile.e == a.E && a.lora_D;  // the shared expert's precomputed deltas
      const bool any_lora = Bsrc != nullptr;
      if (dtile) {  // [token][128 rows] fp16 into the LoRA staging area, every load in flight at once
        const uint16_t* src = a.lora_D + static_cast<size_t>(tile.row0 - a.lora_D_row0) * a.lora_D_ld + tile.mt * BM;
#pragma unroll 1
        for (int i0 = et; i0 < BN * 16; i0 += 4 * kEpi) {  // four 16-byte loads in flight per thread
          uint4 x[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = i0 + q * kEpi, t = i >> 4, ch = i & 15;
            if (t < tile.n) x[q] = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * a.lora_D_ld + ch * 8);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = i0 + q * kEpi;
            if ((i >> 4) < tile.n) reinterpret_cast<uint4*>(lt)[i] = x[q];
          }
        }
      }
      const int rs = (r + 3) & ~3;  // staged t rows are padded with zeros to whole float4s
      if (any_lora) {  // gate and up rows read different t arrays on SwiGLU tiles: even rows t1, odd rows t2
        const int tn = tile.n * rs;
        const float* g1 = a.lora_t1 + static_cast<size_t>(tile.row0) * r;
        const float* g2 = swiglu && a.lora_t2 ? a.lora_t2 + static_cast<size_t>(tile.row0) * r : nullptr;
#pragma unroll 1
        for (int i0 = et; i0 < tn; i0 += 4 * kEpi) {  // four loads of each set in flight per thread
          float x1[4], x2[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = i0 + q * kEpi, t = i / rs, j = i - t * rs;
            const bool in = i < tn && j < r;
            x1[q] = in ? g1[t * r + j] : 0.f;
            x2[q] = in && g2 ? g2[t * r + j] : 0.f;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = i0 + q * kEpi;
            if (i < tn) {
              lt[i] = x1[q];
              if (swiglu) lt[BN * 32 + i] = x2[q];
            }
          }
        }
      }
      if (!swiglu && tile.e < a.E && a.row_scale)
        for (int i = et; i < tile.n; i += kEpi) rsc[i] = a.row_scale[tile.row0 + i];
      if (any_lora) {  // the rows' LoRA B values, read once per tile (consecutive threads: consecutive i of a row)
        for (int i = et; i < BM * r; i += kEpi) {
          const int row = i / r, j = i - row * r, oo = tile.mt * BM + row;
          bls[j * BM + row] = a.lora_scale * half_bits_to_float(Bsrc[static_cast<size_t>(oo) * r + j]);
        }
      }
      // the epilogue warps leave together (they meet at named barriers below)
      if (epi_any(!bar_wait(acc_full + ab, parity(it, 2), a.timeout_ns))) {
        fail = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t taddr = tmem + static_cast<uint32_t>(ab * BN) + ((static_cast<uint32_t>(quad) * 32u) << 16);
      const float* ltr = lt + (up ? BN * 32 : 0);
      bool range_bad = false;  // a SwiGLU output fp16 cannot hold: MOE_ERR_RANGE
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {  // 16 columns at a time: fewer live registers
        const int c0 = 64 * chalf + 16 * blk;
        float v[16];
        const bool live = c0 < tile.n;
        if (live) tmem_ld16(taddr + c0, v);
        if (blk == 3) {  // the accumulator is read: release it for the tile after next
          asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
          __syncwarp();
          if (lane == 0) bar_arrive(acc_empty + ab);
        }
        if (live && dtile) {  // + the shared expert's delta of this row and token
          const uint16_t* ds = reinterpret_cast<const uint16_t*>(lt);
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (c0 + t < tile.n) v[t] += half_bits_to_float(ds[(c0 + t) * BM + L]);
        }
        if (live && Bsrc) {  // unmerged LoRA: + scale * B[row] . t[token]
#pragma unroll 1
          for (int i = 0; i < r; ++i) {
            const float bi = bls[i * BM + L];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const int tt = c0 + t < tile.n ? c0 + t : tile.n - 1;
              v[t] = fmaf(bi, ltr[tt * rs + i], v[t]);
            }
          }
        }
        if (swiglu) {
          const int col = pair_pos(L >> 1);  // SwiGLU outputs in pair order (the down GEMM's token operand)
          if (live) {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const float partner = __shfl_xor_sync(0xffffffffu, v[t], 1);
              if (!up && c0 + t < tile.n) {
                const float hv = __fdividef(v[t], 1.0f + __expf(-v[t])) * partner;  // fp16 result: fast SiLU
                range_bad |= !(fabsf(hv) <= kF16Max);
                stage[(c0 + t) * 64 + col] = __half_as_ushort(__float2half_rn(hv));
              }
            }
          }
        } else {
          const bool scaled = tile.e < a.E && a.row_scale;
          if (live) {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              if (c0 + t < tile.n) {
                const float xv = scaled ? v[t] * rsc[c0 + t] : v[t];
                stage[(c0 + t) * 128 + L] = __half_as_ushort(__float2half_rn(xv));
              }
            }
          }
        }
      }
      if (swiglu) {
        if (range_bad) report(a.err, 6);
        epi_sync();
        for (int i = et; i < tile.n * 8; i += kEpi) {
          const int t = i >> 3, ch = i & 7;
          *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(tile.row0 + t) * a.out_ld + tile.mt * 64 + ch * 8) =
              reinterpret_cast<const uint4*>(stage + t * 64)[ch];
        }
      } else {
        epi_sync();
        for (int i = et; i < tile.n * 16; i += kEpi) {
          const int t = i >> 4, ch = i & 15;
          *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(tile.row0 + t) * a.out_ld + tile.mt * BM + ch * 8) =
              reinterpret_cast<const uint4*>(stage + t * 128)[ch];
        }
      }
      epi_sync();  // staging buffers are free for the next tile
    }
  }
  if (fail) report(a.err, 5);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

}  // namespace gg3
}  // namespace moe
