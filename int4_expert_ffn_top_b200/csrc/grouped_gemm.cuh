// Grouped GEMM on the 5th-generation tensor cores (tcgen05) for many-token
// batches (prefill): per expert bucket, D[o][t] = sum_k W[o][k] * X[t][k] with
// the expert's weight rows as the MMA M operand and the bucket's tokens as the
// N operand ("swap AB": buckets are often far smaller than 128 tokens, the
// weight rows never are).
//
// Per CTA one tile: 128 weight rows x up to 128 tokens, K in steps of 64 (one
// quantisation group per step), 2-stage shared-memory pipeline:
//  * warps 0-3 dequantise the int4 row records of the tile (w = q*s + b, one
//    fp16 rounding) straight into the 128-byte-swizzled K-major layout the MMA
//    reads, one row per thread;
//  * warp 4 loads the token tile with a 2-D TMA copy (128-byte swizzle);
//  * warp 5 issues tcgen05.mma (kind::f16, fp32 accumulator in TMEM) from one
//    elected thread and commits stage release / accumulator-ready mbarriers;
//  * warps 0-3 then read the accumulator with tcgen05.ld and run the epilogue
//    (SwiGLU for gate/up, gating-weight scaling for down, unmerged LoRA
//    deltas), staging through shared memory for coalesced stores.
// Every wait is bounded; a wait that runs out stops the CTA from issuing more
// copies or MMAs, lets what it issued finish (bounded) and records
// MOE_ERR_TIMEOUT in the error word.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {
namespace gg {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 64;
// Two stages keep a CTA at 66 KB of shared memory, so two CTAs share an SM:
// twice the dequantising warps in flight per SM, which the weight stream needs
// more than a deeper per-CTA pipeline (one layer's expert forward at 3,328
// tokens: 1.53 ms with four stages and one CTA per SM, 0.98 ms with this).
constexpr int STAGES = 2;
constexpr int kThreads = 192;
constexpr int A_STAGE = BM * BK * 2;  // 16 KB
constexpr int B_STAGE = BN * BK * 2;  // 16 KB
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE) + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 128;

struct Tile {
  int e;     // expert id; E = the shared expert
  int mt;    // m-tile (128 weight rows)
  int row0;  // first row of the token operand
  int n;     // tokens in the tile (1..128)
};

enum Epi { EPI_SWIGLU = 0, EPI_DOWN = 1 };

struct Args {
  const Tile* tiles;
  const int* n_tiles;
  const uint8_t* pool;
  int64_t stride;
  const uint8_t* shared_block;
  int E;
  int K;         // reduction length (H for gate/up, I for down)
  int64_t a_off; // byte offset of the weight matrix in an expert block
  int a_rec;     // bytes of one row record of that matrix
  int epi;
  uint16_t* out;  // fp16 rows of the output
  int out_ld;     // elements per output row
  const float* row_scale;  // EPI_DOWN, routed rows: multiplier per token row (gating weight), or null
  // unmerged LoRA in the epilogue: value[o][t] += lora_scale * sum_i B[o'][i] * t[row][i]
  const uint16_t* lora_B1;  // SwiGLU: gate rows (o' = j); DOWN: rows o (shared) -- [*][r]
  const float* lora_t1;     // [row][r]
  const uint16_t* lora_B2;  // SwiGLU: up rows
  const float* lora_t2;
  const uint16_t* lora_Bex; // DOWN, routed: per-expert B [E][H][r] (t from lora_t1, indexed by row)
  int lora_r;
  float lora_scale;
  int* err;
  long long timeout_ns;
  int drop_tile;  // test hook: the CTA of this tile never marks its first operand stage full (-1: off)
};

MOE_DEV uint32_t sa(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

MOE_DEV long long gtime() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

MOE_DEV void bar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sa(b)), "r"(count));
}

MOE_DEV bool bar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(sa(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

MOE_DEV bool bar_wait(uint64_t* b, uint32_t parity, long long timeout_ns) {
  if (bar_test(b, parity)) return true;
  const long long deadline = gtime() + timeout_ns;
  for (int it = 1;; ++it) {
    if (bar_test(b, parity)) return true;
    if ((it & 63) == 0 && gtime() > deadline) return false;
  }
}

MOE_DEV void bar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sa(b)) : "memory");
}

MOE_DEV void bar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sa(b)), "r"(bytes) : "memory");
}

MOE_DEV void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(sa(dst)),
      "l"(map), "r"(x), "r"(y), "r"(sa(bar))
      : "memory");
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
MOE_DEV uint64_t smem_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);          // start address
  d |= static_cast<uint64_t>(1u) << 16;                         // leading byte offset (unused for swizzled K-major)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                 // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;                         // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                         // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 accumulator, M = 128, N = n.
MOE_DEV uint32_t instr_desc(int n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | ((128u >> 4) << 24);
}

MOE_DEV void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

MOE_DEV void mma_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(sa(b)) : "memory");
}

// 32 consecutive accumulator columns of this warp's 32 TMEM lanes -> 32 registers per thread.
// The wait is part of the same asm statement: the outputs are defined only once
// the asynchronous load has landed, so no use of them can be scheduled earlier.
MOE_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,"
      "%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// One int4 word (nibble j at bits 4j) -> 8 fp16 weights q*s + b in natural order.
MOE_DEV uint4 dequant_word(uint32_t w, __half2 s2, __half2 b2) {
  uint32_t q[4];
  int4_word_to_h2(w, q);  // (q_j - 8, q_{j+4} - 8), j = 0..3
  const __half2 k8 = __half2half2(__ushort_as_half(0x4800));  // 8
  uint32_t v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = h2_bits(__hfma2(__hadd2(as_h2(q[j]), k8), s2, b2));  // (w_j, w_{j+4})
  return make_uint4(prmt(v[0], v[1], 0x5410u), prmt(v[2], v[3], 0x5410u), prmt(v[0], v[1], 0x7632u),
                    prmt(v[2], v[3], 0x7632u));
}

__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b,
                                                                   const __grid_constant__ Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = sm;
  uint8_t* smB = sm + STAGES * A_STAGE;
  uint64_t* full_a = reinterpret_cast<uint64_t*>(sm + STAGES * (A_STAGE + B_STAGE));
  uint64_t* full_b = full_a + STAGES;
  uint64_t* empty = full_b + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

  if (static_cast<int>(blockIdx.x) >= *a.n_tiles) return;
  const Tile tile = a.tiles[blockIdx.x];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KT = a.K / BK;
  const uint8_t* blk = tile.e < a.E ? a.pool + static_cast<int64_t>(tile.e) * a.stride : a.shared_block;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      bar_init(full_a + s, 128);
      bar_init(full_b + s, 1);
      bar_init(empty + s, 1);
    }
    bar_init(acc_full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sa(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  int fail = 0;

  if (warp < 4) {
    // ---------------------------------------------------------------- dequantising producers (one row each)
    const int r = tid;
    const uint8_t* row = blk + a.a_off + static_cast<int64_t>(tile.mt * BM + r) * a.a_rec;
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(row + a.K / 2);
    const uint16_t* bi = sc + KT;
    uint8_t* dst_row = smA + (r >> 3) * 1024 + (r & 7) * 128;
    uint4 c0 = ldg_stream(row), c1 = ldg_stream(row + 16);
    uint16_t s_raw = sc[0], b_raw = bi[0];
#pragma unroll 1
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % STAGES;
      const uint32_t ph = (kt / STAGES) & 1u;
      const uint4 w0 = c0, w1 = c1;
      const __half2 s2 = __half2half2(__ushort_as_half(s_raw)), b2 = __half2half2(__ushort_as_half(b_raw));
      if (kt + 1 < KT) {  // prefetch the next group
        c0 = ldg_stream(row + (kt + 1) * 32);
        c1 = ldg_stream(row + (kt + 1) * 32 + 16);
        s_raw = sc[kt + 1];
        b_raw = bi[kt + 1];
      }
      if (!bar_wait(empty + s, ph ^ 1u, a.timeout_ns)) {  // never overwrite a stage the MMA may still read
        fail = 1;
        break;
      }
      uint8_t* d = dst_row + s * A_STAGE;
      const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(d + ((c ^ (r & 7)) << 4)) = dequant_word(ws[c], s2, b2);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (!(kt == 0 && r == 0 && static_cast<int>(blockIdx.x) == a.drop_tile)) bar_arrive(full_a + s);
    }
  } else if (warp == 4) {
    // ---------------------------------------------------------------- token tiles by TMA
    if (lane == 0) {
      int issued = 0;
#pragma unroll 1
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1u;
        if (!bar_wait(empty + s, ph ^ 1u, a.timeout_ns)) {
          fail = 1;
          break;
        }
        bar_expect_tx(full_b + s, B_STAGE);
        tma_load_2d(smB + s * B_STAGE, &tmap_b, kt * BK, tile.row0, full_b + s);
        issued = kt + 1;
      }
      if (fail)  // let the loads already issued land before the CTA can exit
#pragma unroll 1
        for (int kt = issued - STAGES > 0 ? issued - STAGES : 0; kt < issued; ++kt)
          bar_wait(full_b + kt % STAGES, (kt / STAGES) & 1u, a.timeout_ns);
    }
  } else {
    // ---------------------------------------------------------------- MMA issue (one thread)
    if (lane == 0) {
      const int n_mma = (tile.n + 15) & ~15;
      const uint32_t idesc = instr_desc(n_mma);
#pragma unroll 1
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1u;
        if (!bar_wait(full_a + s, ph, a.timeout_ns) || !bar_wait(full_b + s, ph, a.timeout_ns)) {
          fail = 1;  // issue nothing more; the commit below still tracks what was issued
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = sa(smA + s * A_STAGE), b0 = sa(smB + s * B_STAGE);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_f16(tmem, smem_desc(a0 + kk * 32), smem_desc(b0 + kk * 32), idesc, (kt | kk) != 0);
        mma_commit(empty + s);
      }
      mma_commit(acc_full);
    }
  }

  if (warp < 4) {
    // ---------------------------------------------------------------- epilogue
    if (!bar_wait(acc_full, 0, a.timeout_ns)) fail = 1;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const int L = tid;  // TMEM lane = tile row
    const int o = tile.mt * BM + L;
    uint16_t* stage = reinterpret_cast<uint16_t*>(sm);  // reuse the pipeline buffers (all MMAs are done)
    const int r = a.lora_r;
    if (a.epi == EPI_SWIGLU) {
      bool range_bad = false;  // a SwiGLU output fp16 cannot hold: MOE_ERR_RANGE
      const bool up = (L & 1) != 0;
      const int j = o >> 1;
      // LoRA B row of this output row (gate or up), r <= 32 values
      float Bl[32];
      const bool sh = tile.e == a.E;  // the shared expert's gate/up carry LoRA deltas
      const uint16_t* Bsrc = sh ? (up ? a.lora_B2 : a.lora_B1) : nullptr;
      const float* tsrc = up ? a.lora_t2 : a.lora_t1;
#pragma unroll
      for (int i = 0; i < 32; ++i) Bl[i] = (Bsrc && i < r) ? half_bits_to_float(Bsrc[static_cast<size_t>(j) * r + i]) : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < tile.n; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + ((static_cast<uint32_t>(warp) * 32u) << 16) + c0, v);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          float x = v[t];
          if (Bsrc && c0 + t < tile.n) {
            const float* tv = tsrc + static_cast<size_t>(tile.row0 + c0 + t) * r;
            float d = 0.f;
            for (int i = 0; i < r; ++i) d = fmaf(Bl[i], tv[i], d);
            x = fmaf(a.lora_scale, d, x);
          }
          const float partner = __shfl_xor_sync(0xffffffffu, x, 1);
          if (!up && c0 + t < tile.n) {
            const float hv = silu(x) * partner;
            range_bad |= !(fabsf(hv) <= kF16Max);
            stage[(c0 + t) * 64 + (L >> 1)] = __half_as_ushort(__float2half_rn(hv));
          }
        }
      }
      if (range_bad) report(a.err, 6);
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // coalesced stores: row (row0 + t), columns [mt*64, mt*64 + 64)
      for (int i = tid; i < tile.n * 8; i += 128) {
        const int t = i >> 3, ch = i & 7;
        *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(tile.row0 + t) * a.out_ld + tile.mt * 64 + ch * 8) =
            reinterpret_cast<const uint4*>(stage + t * 64)[ch];
      }
    } else {
      float Bl[32];
      const uint16_t* Bsrc = tile.e < a.E ? (a.lora_Bex ? a.lora_Bex + static_cast<size_t>(tile.e) * (a.out_ld) * r : nullptr)
                                          : a.lora_B1;
#pragma unroll
      for (int i = 0; i < 32; ++i) Bl[i] = (Bsrc && i < r) ? half_bits_to_float(Bsrc[static_cast<size_t>(o) * r + i]) : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < tile.n; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + ((static_cast<uint32_t>(warp) * 32u) << 16) + c0, v);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          if (c0 + t < tile.n) {
            const int row = tile.row0 + c0 + t;
            float x = v[t];
            if (Bsrc) {
              const float* tv = a.lora_t1 + static_cast<size_t>(row) * r;
              float d = 0.f;
              for (int i = 0; i < r; ++i) d = fmaf(Bl[i], tv[i], d);
              x = fmaf(a.lora_scale, d, x);
            }
            if (tile.e < a.E && a.row_scale) x *= a.row_scale[row];
            stage[(c0 + t) * 128 + L] = __half_as_ushort(__float2half_rn(x));
          }
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      for (int i = tid; i < tile.n * 16; i += 128) {
        const int t = i >> 4, ch = i & 15;
        *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(tile.row0 + t) * a.out_ld + tile.mt * BM + ch * 8) =
            reinterpret_cast<const uint4*>(stage + t * 128)[ch];
      }
    }
  }
  if (fail) report(a.err, 5);
  if (warp == 5 && lane == 0 && fail)  // the accumulator must be idle before its columns are released
    bar_wait(acc_full, 0, a.timeout_ns);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 5) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

}  // namespace gg
}  // namespace moe
