// Supporting kernels of the many-token (grouped GEMM) expert path: parallel
// deterministic token buckets, the permuted fp16 token matrix, the device-side
// tile list, the shared expert's 8-bit gate and LoRA-A products and its per-token
// LoRA deltas, the routed adapters' LoRA-A products, and the gather-combine.
#pragma once

#include "grouped_gemm3.cuh"
#include "layer_kernels.cuh"

namespace moe {
namespace pf {

constexpr int kChunk = 256;  // slots per bucketing block (= block size)

// Per-block expert histograms of the clamped indices (integer counts: order-free).
__global__ void __launch_bounds__(kChunk) bucket_count_kernel(const int32_t* __restrict__ idx_in, int TK, int E,
                                                              int32_t* __restrict__ idx, int32_t* __restrict__ blockhist) {
  __shared__ int h[256];
  for (int e = threadIdx.x; e < E; e += kChunk) h[e] = 0;
  __syncthreads();
  const int s = blockIdx.x * kChunk + threadIdx.x;
  if (s < TK) {
    int v = idx_in[s];
    v = v < 0 ? 0 : (v >= E ? E - 1 : v);
    idx[s] = v;
    atomicAdd(&h[v], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kChunk) blockhist[static_cast<size_t>(blockIdx.x) * E + e] = h[e];
}

// One block: expert offsets (exclusive scan of the totals) and, per block and
// expert, the first sorted position of that block's slots (in place).  Thread e
// owns expert e; the scan over experts is a warp-shuffle scan plus the warps'
// totals, and each thread reads its column of the block histograms 8 blocks at
// a time before writing them back.
__global__ void __launch_bounds__(256) bucket_scan_kernel(int nblk, int E, int32_t* __restrict__ blockhist,
                                                          int32_t* __restrict__ count, int32_t* __restrict__ offset) {
  __shared__ int wsum[8];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  int t = 0;
  if (e < E) {
#pragma unroll 8
    for (int b = 0; b < nblk; ++b) t += blockhist[static_cast<size_t>(b) * E + e];
  }
  int incl = t;  // inclusive scan within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int excl = incl - t;
  for (int w = 0; w < warp; ++w) excl += wsum[w];
  if (e < E) {
    count[e] = t;
    offset[e] = excl;
    if (e == E - 1) offset[E] = excl + t;
    int run = excl;
#pragma unroll 1
    for (int b0 = 0; b0 < nblk; b0 += 8) {
      int c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = b0 + i < nblk ? blockhist[static_cast<size_t>(b0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (b0 + i < nblk) {
          blockhist[static_cast<size_t>(b0 + i) * E + e] = run;
          run += c[i];
        }
      }
    }
  }
}

// Stable placement: the rank of a slot among equal experts of its block
// (warp match + per-warp counts) plus the block's base position.
__global__ void __launch_bounds__(kChunk) bucket_place_kernel(const int32_t* __restrict__ idx, int TK, int E,
                                                              const int32_t* __restrict__ base, int32_t* __restrict__ perm,
                                                              int32_t* __restrict__ inv, int32_t* __restrict__ perm_out) {
  __shared__ int wcnt[kChunk / 32][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (kChunk / 32) * 256; i += kChunk) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int s = blockIdx.x * kChunk + threadIdx.x;
  const bool act = s < TK;
  const int e = act ? idx[s] : -1 - lane;
  const unsigned m = __match_any_sync(0xffffffffu, e);
  const int rank_w = __popc(m & ((1u << lane) - 1u));
  if (act && rank_w == 0) wcnt[warp][e] = __popc(m);
  __syncthreads();
  if (act) {
    int pos = base[static_cast<size_t>(blockIdx.x) * E + e] + rank_w;
    for (int w2 = 0; w2 < warp; ++w2) pos += wcnt[w2][e];
    perm[pos] = s;
    inv[s] = pos;
    if (perm_out) perm_out[pos] = s;
  }
}

// Token operand rows in fp16: rows [0, TK) are the slots in bucket order (the
// slot's token), rows [TK, TK+T) the tokens in order (shared expert).  Also the
// gating weight of each sorted slot.  Each 8-element block is stored in pair
// order (u_j, u_{j+4}), j = 0..3, the K order of the dequantised weight tiles.
// Activations fp16 cannot hold (|u| > 65504 or not finite) report MOE_ERR_RANGE
// into err (checked on the shared-expert rows, which hold every token once).
// One warp per row, 8 rows per CTA; a lane's H / 256 16-byte loads are all issued before its stores.
template <int H>
__global__ void __launch_bounds__(256) permute_kernel(const uint16_t* __restrict__ u, int T, int K,
                                                      const int32_t* __restrict__ perm, const float* __restrict__ w,
                                                      uint16_t* __restrict__ X, float* __restrict__ w_pos, int* err) {
  constexpr int NV = H / 256;
  const int lane = threadIdx.x & 31, row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int TK = T * K;
  if (row >= TK + T) return;  // whole warps
  int tok;
  if (row < TK) {
    const int slot = perm[row];
    tok = slot / K;
    if (lane == 0) w_pos[row] = w[slot];
  } else {
    tok = row - TK;
  }
  const uint4* src = reinterpret_cast<const uint4*>(u + static_cast<size_t>(tok) * H);
  uint4* dst = reinterpret_cast<uint4*>(X + static_cast<size_t>(row) * H);
  uint4 v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = src[lane + 32 * i];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint32_t vw[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    uint16_t e[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint16_t lo = static_cast<uint16_t>(vw[j] & 0xffffu), hi = static_cast<uint16_t>(vw[j] >> 16);
      bad |= !(fabsf(bf16_bits_to_float(lo)) <= kF16Max) || !(fabsf(bf16_bits_to_float(hi)) <= kF16Max);
      e[2 * j] = bf16_to_f16_bits(lo);
      e[2 * j + 1] = bf16_to_f16_bits(hi);
    }
    dst[lane + 32 * i] =
        make_uint4(e[0] | (static_cast<uint32_t>(e[4]) << 16), e[1] | (static_cast<uint32_t>(e[5]) << 16),
                   e[2] | (static_cast<uint32_t>(e[6]) << 16), e[3] | (static_cast<uint32_t>(e[7]) << 16));
  }
  if (row >= TK && __any_sync(0xFFFFFFFFu, bad) && lane == 0) report(err, 6);
}

// Tile lists of both GEMMs: per expert (then the shared expert) its token
// n-tiles, m-tiles innermost, so CTAs that share a token tile run together.
// One block per expert (block E: the shared expert): the block sums the n-tile
// counts of the experts before it, then writes its tiles with all threads.
__global__ void __launch_bounds__(128) tile_list_kernel(const int32_t* __restrict__ count,
                                                        const int32_t* __restrict__ offset, int E, int T, int K,
                                                        int mt_gu, int mt_dn, tc::Tile* __restrict__ tiles_gu,
                                                        tc::Tile* __restrict__ tiles_dn, int* __restrict__ n_tiles) {
  constexpr int BN = gg3::BN;
  __shared__ int red[4];
  const int e = blockIdx.x;  // 0..E
  int before = 0;
  for (int i = threadIdx.x; i < e; i += blockDim.x) before += (count[i] + BN - 1) / BN;
  before = __reduce_add_sync(0xffffffffu, before);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = before;
  __syncthreads();
  const int start = red[0] + red[1] + red[2] + red[3];
  const int n = e < E ? count[e] : T;
  const int nt = (n + BN - 1) / BN;
  const int base = e < E ? offset[e] : T * K;
  if (e == E && threadIdx.x == 0) {
    n_tiles[0] = (start + nt) * mt_gu;
    n_tiles[1] = (start + nt) * mt_dn;
  }
  const int mt = mt_gu > mt_dn ? mt_gu : mt_dn;
  for (int i = threadIdx.x; i < nt * mt; i += blockDim.x) {
    const int q = i / mt, m = i % mt, n0 = q * BN, nn = min(BN, n - n0), t = start + q;
    if (m < mt_dn) tiles_dn[t * mt_dn + m] = tc::Tile{e, m, base + n0, nn};
    if (m < mt_gu) tiles_gu[t * mt_gu + m] = tc::Tile{e, m, base + n0, nn};
  }
}

// Shared expert's gate and gate/up LoRA-A products for many tokens, in one pass over u:
//   g[t] = sigmoid(w . u_t), w the 8-bit gate row (affine groups of 64): per group s * sum (q - 128) u + (b + 128 s) * sum u;
//   the LoRA-A products t1 = A_gate u_t and t2 = A_up u_t (r values each; a projection without adapter gets
//   zeros) into tv[t] = (t1, t2), from which lora_delta_kernel forms the unmerged deltas the gate/up GEMM adds.
// A CTA takes 16 tokens and copies their rows of u into shared memory (16-byte asynchronous copies, all in flight
// at once; rows padded by 64 bytes so that a warp's reads hit distinct banks).  Its 8 warps split the input
// dimension into 32-wide chunks (warp w: chunks w, w + 8, ...), and the warps' partial sums are added in warp
// order at the end.  The LoRA-A products run on tensor cores as tf32 m16n8k8 MMAs: bf16 u and fp16 A are exact in
// tf32, so the products are exact and only the fp32 accumulation rounds.  Within a chunk, lane (g, q) supplies
// inputs 8q + 2s and 8q + 2s + 1 as the MMA's k = q and k = q + 4 of step s, for both operands alike.
constexpr int kStTok = 16, kStWarps = 8;
inline int shared_tokens_nt(int r) { return r <= 0 ? 0 : (2 * r <= 16 ? 2 : (2 * r <= 32 ? 4 : 8)); }
inline int shared_tokens_smem(int H, int nt) {
  const int stage = kStTok * (2 * H + 64), red = kStWarps * kStTok * 8 * nt * 4;
  return stage > red ? stage : red;
}

MOE_DEV void mma_tf32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[t0 + tok][o] = fp16(scale * B_o . t[tok]) for the tokens of a 16-token block and the outputs
// o_begin <= o < o_end (a row of D holds n_out outputs), t[tok] = tS[j][tok] (j < r).
// pairs = false: B_o is row o of B_even ([n_out][r]).  pairs = true (the
// interleaved gate/up rows): B_o is row o / 2 of B_even for even o and of B_odd for odd o (each [n_out / 2][r]),
// and the odd rows read t from tS[r + j].  A null B gives zeros.  Two outputs per thread and pass, all 16
// tokens; a B row is read 8 ranks per 16-byte load when r is a multiple of 8.
MOE_DEV void lora_delta_rows(const float (*tS)[kStTok], bool pairs, int r, int t0, int T, int n_out, int o_begin,
                             int o_end, const uint16_t* __restrict__ B_even, const uint16_t* __restrict__ B_odd,
                             float scale, uint16_t* __restrict__ D) {
  const bool vec = (r & 7) == 0;
  // two outputs blockDim.x apart per pass (same parity: blockDim.x and o_begin are even), their B loads together
#pragma unroll 1
  for (int o0 = o_begin + threadIdx.x; o0 < o_end; o0 += 2 * blockDim.x) {
    const bool odd = pairs && (o0 & 1);
    const uint16_t* B = odd ? B_odd : B_even;
    const uint16_t* src[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int o = o0 + m * blockDim.x;
      src[m] = (B && o < o_end) ? B + static_cast<size_t>(pairs ? o >> 1 : o) * r : nullptr;
    }
    const int js = odd ? r : 0;
    float acc[2][kStTok];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int k = 0; k < kStTok; ++k) acc[m][k] = 0.f;
#pragma unroll 1
    for (int j0 = 0; (src[0] || src[1]) && j0 < r; j0 += 8) {
      float b[2][8];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        if (vec) {
          const uint4 w = src[m] ? *reinterpret_cast<const uint4*>(src[m] + j0) : make_uint4(0, 0, 0, 0);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(as_h2(ww[e]));
            b[m][2 * e] = f.x;
            b[m][2 * e + 1] = f.y;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) b[m][e] = (src[m] && j0 + e < r) ? half_bits_to_float(src[m][j0 + e]) : 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (j0 + e >= r) break;
        const float4* tr = reinterpret_cast<const float4*>(tS[js + j0 + e]);
#pragma unroll
        for (int q = 0; q < kStTok / 4; ++q) {
          const float4 x = tr[q];
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            acc[m][4 * q] = fmaf(b[m][e], x.x, acc[m][4 * q]);
            acc[m][4 * q + 1] = fmaf(b[m][e], x.y, acc[m][4 * q + 1]);
            acc[m][4 * q + 2] = fmaf(b[m][e], x.z, acc[m][4 * q + 2]);
            acc[m][4 * q + 3] = fmaf(b[m][e], x.w, acc[m][4 * q + 3]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int o = o0 + m * blockDim.x;
      if (o >= o_end) continue;
#pragma unroll
      for (int k = 0; k < kStTok; ++k)
        if (t0 + k < T)
          D[static_cast<size_t>(t0 + k) * n_out + o] = __half_as_ushort(__float2half_rn(scale * acc[m][k]));
    }
  }
}

template <int NT>  // 8-row tiles of the 2r LoRA rows (gate rows, then up rows); 0: the gate only
__global__ void __launch_bounds__(256) shared_tokens_kernel(const uint16_t* __restrict__ u, int T, int H,
                                                            const uint8_t* __restrict__ rec, float* __restrict__ g,
                                                            int r, const uint16_t* __restrict__ A_gate,
                                                            const uint16_t* __restrict__ A_up,
                                                            float* __restrict__ tv) {
  constexpr int NTa = NT > 0 ? NT : 1, NC = 8 * NTa;
  extern __shared__ __align__(16) uint8_t st_smem[];
  __shared__ float gred[kStWarps][kStTok];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gi = lane >> 2, q = lane & 3;
  const int t0 = blockIdx.x * kStTok, ld = 2 * H + 64;  // staged row stride in bytes
  // stage the 16 token rows (rows past T are zeros)
  const int n16 = H / 8;  // 16-byte pieces per row
  for (int i = threadIdx.x; i < kStTok * n16; i += blockDim.x) {
    const int row = i / n16, piece = i - row * n16;
    uint8_t* dst = st_smem + row * ld + piece * 16;
    if (t0 + row < T)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                   "l"(u + static_cast<size_t>(t0 + row) * H + piece * 8)
                   : "memory");
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + H);
  const uint16_t* arow[NTa];
#pragma unroll
  for (int n = 0; n < NTa; ++n) {
    const int j = 8 * n + gi;
    arow[n] = NT == 0 ? nullptr
                      : (j < r ? (A_gate ? A_gate + static_cast<size_t>(j) * H : nullptr)
                               : (j < 2 * r && A_up ? A_up + static_cast<size_t>(j - r) * H : nullptr));
  }
  // per-chunk global inputs: the gate codes and scales, the A fragments; fetched one chunk ahead
  struct Pre {
    uint2 qc;
    uint16_t s, b;
    uint4 a[NTa];
  };
  auto fetch = [&](int c, Pre& p) {
    const int k = c * 32 + 8 * q;
    p.qc = *reinterpret_cast<const uint2*>(rec + k);
    p.s = sc[k >> 6];
    p.b = sc[H / 64 + (k >> 6)];
#pragma unroll
    for (int n = 0; n < NTa; ++n)
      p.a[n] = (NT > 0 && arow[n]) ? *reinterpret_cast<const uint4*>(arow[n] + k) : make_uint4(0, 0, 0, 0);
  };
  float acc[NTa][4];
#pragma unroll
  for (int n = 0; n < NTa; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float ga = 0.f, gb = 0.f;  // gate partials of tokens gi and gi + 8
  const int nch = H / 32;
  Pre cur, nxt;
  if (warp < nch) fetch(warp, cur);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
#pragma unroll 1
  for (int c = warp; c < nch; c += kStWarps) {
    if (c + kStWarps < nch) fetch(c + kStWarps, nxt);
    const int k = c * 32 + 8 * q;
    const uint4 xa = *reinterpret_cast<const uint4*>(st_smem + gi * ld + 2 * k);
    const uint4 xb = *reinterpret_cast<const uint4*>(st_smem + (gi + 8) * ld + 2 * k);
    // u as fp32 bit patterns (bf16 << 16): element 2e is the low half of word e
    const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w}, wb[4] = {xb.x, xb.y, xb.z, xb.w};
    uint32_t ua[8], ub[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      ua[2 * e] = wa[e] << 16;
      ua[2 * e + 1] = wa[e] & 0xFFFF0000u;
      ub[2 * e] = wb[e] << 16;
      ub[2 * e + 1] = wb[e] & 0xFFFF0000u;
    }
    {  // gate
      float da = 0.f, sa = 0.f, db = 0.f, sb = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t w = i < 4 ? cur.qc.x : cur.qc.y;
        const float qv = static_cast<float>(static_cast<int>((w >> (8 * (i & 3))) & 0xFFu) - 128);
        const float x = __uint_as_float(ua[i]), y = __uint_as_float(ub[i]);
        da = fmaf(qv, x, da);
        sa += x;
        db = fmaf(qv, y, db);
        sb += y;
      }
      const float s = half_bits_to_float(cur.s), bb = fmaf(128.f, s, half_bits_to_float(cur.b));
      ga += fmaf(s, da, bb * sa);
      gb += fmaf(s, db, bb * sb);
    }
    if (NT > 0) {
#pragma unroll
      for (int n = 0; n < NTa; ++n) {
        const uint32_t aw[4] = {cur.a[n].x, cur.a[n].y, cur.a[n].z, cur.a[n].w};
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          const float2 f = __half22float2(as_h2(aw[st]));
          mma_tf32(acc[n], ua[2 * st], ub[2 * st], ua[2 * st + 1], ub[2 * st + 1], __float_as_uint(f.x),
                   __float_as_uint(f.y));
        }
      }
    }
    cur = nxt;
  }
  ga += __shfl_xor_sync(0xFFFFFFFFu, ga, 1);
  ga += __shfl_xor_sync(0xFFFFFFFFu, ga, 2);
  gb += __shfl_xor_sync(0xFFFFFFFFu, gb, 1);
  gb += __shfl_xor_sync(0xFFFFFFFFu, gb, 2);
  __syncthreads();  // the staged rows are read: the area now holds the warps' partial products
  float* red = reinterpret_cast<float*>(st_smem);  // [warp][token][NC]
  if (q == 0) {
    gred[warp][gi] = ga;
    gred[warp][gi + 8] = gb;
  }
  if (NT > 0) {
#pragma unroll
    for (int n = 0; n < NTa; ++n) {
      float* p = red + (warp * kStTok + gi) * NC + 8 * n + 2 * q;
      p[0] = acc[n][0];
      p[1] = acc[n][1];
      p[8 * NC] = acc[n][2];
      p[8 * NC + 1] = acc[n][3];
    }
  }
  __syncthreads();
  if (threadIdx.x < kStTok && t0 + threadIdx.x < T) {
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < kStWarps; ++w) z += gred[w][threadIdx.x];
    g[t0 + threadIdx.x] = sigmoid(z);
  }
  if (NT > 0) {
    for (int i = threadIdx.x; i < kStTok * NC; i += blockDim.x) {
      const int tok = i / NC, j = i - tok * NC;
      if (j >= 2 * r || t0 + tok >= T) continue;
      float z = 0.f;
#pragma unroll
      for (int w = 0; w < kStWarps; ++w) z += red[(w * kStTok + tok) * NC + j];
      tv[static_cast<size_t>(t0 + tok) * 2 * r + j] = z;
    }
  }
}

// The shared expert's unmerged LoRA deltas from per-token t vectors tv [T][kt] (pairs: kt = 2r, the gate's r
// then the up's r; else kt = r): D[t][o] = fp16(scale * B_o . t_t) for the n_out outputs (lora_delta_rows).
// Grid (token blocks of 16, output blocks of 256); 128 threads, two outputs per thread.
constexpr int kDeltaOut = 256;
__global__ void __launch_bounds__(128) lora_delta_kernel(const float* __restrict__ tv, int T, int r, bool pairs,
                                                         int n_out, const uint16_t* __restrict__ B_even,
                                                         const uint16_t* __restrict__ B_odd, float scale,
                                                         uint16_t* __restrict__ D) {
  __shared__ __align__(16) float tS[64][kStTok];
  const int t0 = blockIdx.x * kStTok, kt = pairs ? 2 * r : r;
  for (int i = threadIdx.x; i < kStTok * kt; i += blockDim.x) {
    const int tok = i / kt, j = i - tok * kt;
    tS[j][tok] = t0 + tok < T ? tv[static_cast<size_t>(t0 + tok) * kt + j] : 0.f;
  }
  __syncthreads();
  const int o_begin = blockIdx.y * kDeltaOut, o_end = o_begin + kDeltaOut < n_out ? o_begin + kDeltaOut : n_out;
  lora_delta_rows(tS, pairs, r, t0, T, n_out, o_begin, o_end, B_even, B_odd, scale, D);
}

// Shared expert's down-projection LoRA-A products for many tokens: tv[t] = A_down h_t (r values), h_t the
// token's SwiGLU output (fp16, pair order within 8-element blocks; A_down [r][I] in natural order), from which
// lora_delta_kernel forms the delta.  A CTA takes 16 tokens: their h rows and the r rows of A_down go to shared
// memory first (16-byte asynchronous copies, all in flight; rows padded by 16 bytes so that the eight lanes of
// a 16-byte load phase, eight tokens, hit distinct banks); a thread then forms one or two of the 16 x r products.
inline int shared_down_lora_smem(int I, int r) { return (kStTok + r) * (2 * I + 16); }
__global__ void __launch_bounds__(256) shared_down_lora_kernel(const uint16_t* __restrict__ h, int T, int I, int r,
                                                               const uint16_t* __restrict__ A_d,
                                                               float* __restrict__ tv) {
  extern __shared__ __align__(16) uint8_t sd_smem[];
  const int t0 = blockIdx.x * kStTok, ld = 2 * I + 16, n16 = I / 8;  // staged row stride in bytes
  for (int i = threadIdx.x; i < (kStTok + r) * n16; i += blockDim.x) {
    const int row = i / n16, piece = i - row * n16;
    uint8_t* dst = sd_smem + row * ld + piece * 16;
    const uint16_t* src = row < kStTok ? (t0 + row < T ? h + static_cast<size_t>(t0 + row) * I : nullptr)
                                       : A_d + static_cast<size_t>(row - kStTok) * I;
    if (src)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                   "l"(src + piece * 8)
                   : "memory");
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  for (int p = threadIdx.x; p < kStTok * r; p += blockDim.x) {
    const int tok = p & (kStTok - 1), j = p / kStTok;
    const uint4* hr = reinterpret_cast<const uint4*>(sd_smem + tok * ld);
    const uint4* ar = reinterpret_cast<const uint4*>(sd_smem + (kStTok + j) * ld);
    float acc = 0.f;
#pragma unroll 4
    for (int c = 0; c < n16; ++c) {
      const uint4 w = ar[c], hv = hr[c];
      acc = dot2_mix(prmt(w.x, w.z, 0x5410u), hv.x, acc);  // A chunk to pair order
      acc = dot2_mix(prmt(w.x, w.z, 0x7632u), hv.y, acc);
      acc = dot2_mix(prmt(w.y, w.w, 0x5410u), hv.z, acc);
      acc = dot2_mix(prmt(w.y, w.w, 0x7632u), hv.w, acc);
    }
    if (t0 + tok < T) tv[static_cast<size_t>(t0 + tok) * r + j] = acc;
  }
}

// The routed down adapters' LoRA-A products on the SwiGLU output rows of the routed slots (rows < TK):
// t[row][i] = A_e[i] . h[row], e the row's expert (A_ex [E][r][I]).  One warp per (row, i); h rows are fp16 in
// pair order, A rows in natural order.
__global__ void __launch_bounds__(kThreads) lora_a_rows_kernel(const uint16_t* __restrict__ h, int I, int TK, int r,
                                                               const uint16_t* __restrict__ A_ex,
                                                               const int32_t* __restrict__ idx,
                                                               const int32_t* __restrict__ perm, float* __restrict__ t) {
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (gw >= TK * r) return;
  const int row = gw / r, i = gw % r;
  const uint16_t* A = A_ex + (static_cast<size_t>(idx[perm[row]]) * r + i) * I;
  const uint16_t* hr = h + static_cast<size_t>(row) * I;
  float acc = 0.f;
  for (int c = lane; c < I / 8; c += 32) {
    const uint4 w = reinterpret_cast<const uint4*>(A)[c];
    const uint4 hv = reinterpret_cast<const uint4*>(hr)[c];
    acc = dot2_mix(prmt(w.x, w.z, 0x5410u), hv.x, acc);  // A chunk to pair order
    acc = dot2_mix(prmt(w.x, w.z, 0x7632u), hv.y, acc);
    acc = dot2_mix(prmt(w.y, w.w, 0x5410u), hv.z, acc);
    acc = dot2_mix(prmt(w.y, w.w, 0x7632u), hv.w, acc);
  }
  acc = warp_reduce(acc);
  if (lane == 0) t[static_cast<size_t>(row) * r + i] = acc;
}

// LoRA-A products of the routed experts' gate and up adapters on the permuted token rows (rows < TK):
// t1[row][i] = A_gate[e][i] . x[row] and t2[row][i] = A_up[e][i] . x[row], e the row's expert.  One warp per
// (row, j < 2r); x rows are fp16 in pair order, A rows in natural order ([E][2][r][H]: gate's, then up's).
__global__ void __launch_bounds__(kThreads) lora_a_gu_rows_kernel(const uint16_t* __restrict__ X, int H, int TK, int r,
                                                                  const uint16_t* __restrict__ A_gu,
                                                                  const int32_t* __restrict__ idx,
                                                                  const int32_t* __restrict__ perm,
                                                                  float* __restrict__ t1, float* __restrict__ t2) {
  const long long gw = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(TK) * 2 * r) return;
  const int row = static_cast<int>(gw / (2 * r)), j = static_cast<int>(gw % (2 * r));
  const uint16_t* A = A_gu + (static_cast<size_t>(idx[perm[row]]) * 2 * r + j) * H;
  const uint16_t* xr = X + static_cast<size_t>(row) * H;
  float acc = 0.f;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 w = reinterpret_cast<const uint4*>(A)[c];
    const uint4 xv = reinterpret_cast<const uint4*>(xr)[c];
    acc = dot2_mix(prmt(w.x, w.z, 0x5410u), xv.x, acc);  // A chunk to pair order
    acc = dot2_mix(prmt(w.x, w.z, 0x7632u), xv.y, acc);
    acc = dot2_mix(prmt(w.y, w.w, 0x5410u), xv.z, acc);
    acc = dot2_mix(prmt(w.y, w.w, 0x7632u), xv.w, acc);
  }
  acc = warp_reduce(acc);
  if (lane == 0) (j < r ? t1 : t2)[static_cast<size_t>(row) * r + (j < r ? j : j - r)] = acc;
}

// out[t] (=, bf16, or +=) sum_k y[inv[t*K+k]] + g[t] * y[TK+t]; the routed rows of
// y already carry their gating weight; k order fixed.
// A thread's K + 1 row loads are all issued before the sum (row ids read once per token); the stores are
// 16-byte vectors when out is 16-byte aligned.
template <int H>
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y, int T, int K,
                                                      const int32_t* __restrict__ inv, const float* __restrict__ g,
                                                      void* __restrict__ out, int out_mode) {
  constexpr int kMaxK = 8;
  const int t = blockIdx.x;
  const int TK = T * K;
  int rows[kMaxK];
#pragma unroll
  for (int k = 0; k < kMaxK; ++k) rows[k] = k < K ? inv[t * K + k] : 0;
  const float gt = g[t];
  const bool vec = (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    uint4 v[kMaxK + 1];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k)
      if (k < K) v[k] = reinterpret_cast<const uint4*>(y + static_cast<size_t>(rows[k]) * H)[c];
    v[kMaxK] = reinterpret_cast<const uint4*>(y + static_cast<size_t>(TK + t) * H)[c];
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
      if (k >= K) break;
      const uint32_t vw[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(as_h2(vw[i]));
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
    {
      const uint32_t vw[4] = {v[kMaxK].x, v[kMaxK].y, v[kMaxK].z, v[kMaxK].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(as_h2(vw[i]));
        acc[2 * i] = fmaf(gt, f.x, acc[2 * i]);
        acc[2 * i + 1] = fmaf(gt, f.y, acc[2 * i + 1]);
      }
    }
    const size_t o = static_cast<size_t>(t) * H + c * 8;
    if (out_mode == 1) {
      uint16_t* ob = reinterpret_cast<uint16_t*>(out) + o;
      uint16_t b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) b[i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i]));
      if (vec) {
        *reinterpret_cast<uint4*>(ob) =
            make_uint4(b[0] | (static_cast<uint32_t>(b[1]) << 16), b[2] | (static_cast<uint32_t>(b[3]) << 16),
                       b[4] | (static_cast<uint32_t>(b[5]) << 16), b[6] | (static_cast<uint32_t>(b[7]) << 16));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) ob[i] = b[i];
      }
    } else {
      float* of = reinterpret_cast<float*>(out) + o;
      if (vec) {
        float4* o4 = reinterpret_cast<float4*>(of);
        float4 x0 = make_float4(acc[0], acc[1], acc[2], acc[3]), x1 = make_float4(acc[4], acc[5], acc[6], acc[7]);
        if (out_mode == 2) {
          const float4 p0 = o4[0], p1 = o4[1];
          x0 = make_float4(p0.x + x0.x, p0.y + x0.y, p0.z + x0.z, p0.w + x0.w);
          x1 = make_float4(p1.x + x1.x, p1.y + x1.y, p1.z + x1.z, p1.w + x1.w);
        }
        o4[0] = x0;
        o4[1] = x1;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) of[i] = out_mode == 2 ? of[i] + acc[i] : acc[i];
      }
    }
  }
}

}  // namespace pf
}  // namespace moe
