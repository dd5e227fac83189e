// Supporting kernels of the many-token (grouped GEMM) expert path: parallel
// deterministic token buckets, the permuted fp16 token matrix, the device-side
// tile list, LoRA-A products for many tokens, and the gather-combine.
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
// expert, the first sorted position of that block's slots (in place).
__global__ void __launch_bounds__(256) bucket_scan_kernel(int nblk, int E, int32_t* __restrict__ blockhist,
                                                          int32_t* __restrict__ count, int32_t* __restrict__ offset) {
  __shared__ int tot[256];
  __shared__ int off[257];
  const int e = threadIdx.x;
  if (e < E) {
    int t = 0;
#pragma unroll 8
    for (int b = 0; b < nblk; ++b) t += blockhist[static_cast<size_t>(b) * E + e];
    tot[e] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < E; ++i) {
      off[i] = run;
      run += tot[i];
    }
    off[E] = run;
  }
  __syncthreads();
  if (e < E) {
    count[e] = tot[e];
    offset[e] = off[e];
    int run = off[e];
    for (int b = 0; b < nblk; ++b) {
      const int c = blockhist[static_cast<size_t>(b) * E + e];
      blockhist[static_cast<size_t>(b) * E + e] = run;
      run += c;
    }
  }
  if (threadIdx.x == 0) offset[E] = off[E];
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
__global__ void __launch_bounds__(256) permute_kernel(const uint16_t* __restrict__ u, int T, int K, int H,
                                                      const int32_t* __restrict__ perm, const float* __restrict__ w,
                                                      uint16_t* __restrict__ X, float* __restrict__ w_pos, int* err) {
  const int row = blockIdx.x;
  const int TK = T * K;
  int tok;
  if (row < TK) {
    const int slot = perm[row];
    tok = slot / K;
    if (threadIdx.x == 0) w_pos[row] = w[slot];
  } else {
    tok = row - TK;
  }
  const uint4* src = reinterpret_cast<const uint4*>(u + static_cast<size_t>(tok) * H);
  uint4* dst = reinterpret_cast<uint4*>(X + static_cast<size_t>(row) * H);
  bool bad = false;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const uint4 v = src[c];
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
    uint16_t e[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t lo = static_cast<uint16_t>(vw[i] & 0xffffu), hi = static_cast<uint16_t>(vw[i] >> 16);
      bad |= !(fabsf(bf16_bits_to_float(lo)) <= kF16Max) || !(fabsf(bf16_bits_to_float(hi)) <= kF16Max);
      e[2 * i] = bf16_to_f16_bits(lo);
      e[2 * i + 1] = bf16_to_f16_bits(hi);
    }
    dst[c] = make_uint4(e[0] | (static_cast<uint32_t>(e[4]) << 16), e[1] | (static_cast<uint32_t>(e[5]) << 16),
                        e[2] | (static_cast<uint32_t>(e[6]) << 16), e[3] | (static_cast<uint32_t>(e[7]) << 16));
  }
  if (bad && row >= TK) report(err, 6);
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

// Shared-expert gate and LoRA-A products for many tokens: g[t], t1[TK+t][i] =
// A_gate[i] . u_t, t2[TK+t][i] = A_up[i] . u_t.  grid (ceil(T / TB), row blocks).
template <int NCH8>  // H / 8
__global__ void __launch_bounds__(kThreads) lora_a_tokens_kernel(const uint16_t* __restrict__ u, int T, int TK, int r,
                                                                 const uint8_t* __restrict__ sg_rec,
                                                                 const uint16_t* __restrict__ A_gate,
                                                                 const uint16_t* __restrict__ A_up, float* __restrict__ g,
                                                                 float* __restrict__ t1, float* __restrict__ t2) {
  // (the activation range is checked by permute_kernel, which reads every token)
  constexpr int H = NCH8 * 8;
  constexpr int SEG8 = (H / 16) < 32 ? (H / 16) : 32;
  extern __shared__ uint4 smem[];
  uint4* us = smem;
  float* sum16 = reinterpret_cast<float*>(us + TB * (H / 8));
  __shared__ int tok[TB];
  const int t0 = blockIdx.x * TB, nt = min(TB, T - t0);
  if (threadIdx.x < TB) tok[threadIdx.x] = t0 + min(static_cast<int>(threadIdx.x), nt - 1);
  __syncthreads();
  stage_tokens(u, H, tok, nt, us, nullptr, sum16, false, nullptr);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.y * kWarps + warp;  // 0: shared gate; 1..r: A_gate; r+1..2r: A_up
  const int nrows = 1 + (A_gate ? r : 0) + (A_up ? r : 0);
  if (row >= nrows) return;
  float acc[TB];
#pragma unroll
  for (int t = 0; t < TB; ++t) acc[t] = 0.f;
  if (row == 0) {
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(sg_rec + H);
    row_int8<H / 16, SEG8>(reinterpret_cast<const uint32_t*>(sg_rec), sc, sc + H / 64, us, sum16, nt, lane % SEG8, acc);
#pragma unroll
    for (int t = 0; t < TB; ++t) acc[t] = seg_reduce<SEG8>(acc[t]);
    if (lane == 0)
      for (int t = 0; t < nt; ++t) g[t0 + t] = sigmoid(acc[t]);
  } else {
    constexpr int SEG = NCH8 < 32 ? NCH8 : 32;
    const int i = row - 1;
    const bool is_gate = A_gate && i < r;
    const int ri = is_gate ? i : (A_gate ? i - r : i);
    const uint16_t* A = is_gate ? A_gate : A_up;
    if (lane < SEG) row_f16<NCH8, SEG>(A + static_cast<size_t>(ri) * H, us, H / 8, nt, lane, acc);
#pragma unroll
    for (int t = 0; t < TB; ++t) acc[t] = seg_reduce<32>(acc[t]);
    if (lane == 0) {
      float* dst = is_gate ? t1 : t2;
      for (int t = 0; t < nt; ++t) dst[static_cast<size_t>(TK + t0 + t) * r + ri] = acc[t];
    }
  }
}

// LoRA-A products on the SwiGLU output rows: t[row][i] = A_row[i] . h[row] with
// A = A_down_shared for rows >= TK, else the routed expert's A (if any).
// One warp per (row, i); h rows are fp16 in pair order, A rows in natural order.
__global__ void __launch_bounds__(kThreads) lora_a_rows_kernel(const uint16_t* __restrict__ h, int I, int TK, int nrows,
                                                               int row_begin, int r, const uint16_t* __restrict__ A_sd,
                                                               const uint16_t* __restrict__ A_ex,
                                                               const int32_t* __restrict__ idx,
                                                               const int32_t* __restrict__ perm, float* __restrict__ t) {
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (gw >= nrows * r) return;
  const int row = row_begin + gw / r, i = gw % r;
  const uint16_t* A;
  if (row >= TK) A = A_sd + static_cast<size_t>(i) * I;
  else A = A_ex + (static_cast<size_t>(idx[perm[row]]) * r + i) * I;
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
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y, int T, int K, int H,
                                                      const int32_t* __restrict__ inv, const float* __restrict__ g,
                                                      void* __restrict__ out, int out_mode) {
  const int t = blockIdx.x;
  const int TK = T * K;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int k = 0; k < K; ++k) {
      const uint4 v = reinterpret_cast<const uint4*>(y + static_cast<size_t>(inv[t * K + k]) * H)[c];
      const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(as_h2(vw[i]));
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
    const float gt = g[t];
    const uint4 v = reinterpret_cast<const uint4*>(y + static_cast<size_t>(TK + t) * H)[c];
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(as_h2(vw[i]));
      acc[2 * i] = fmaf(gt, f.x, acc[2 * i]);
      acc[2 * i + 1] = fmaf(gt, f.y, acc[2 * i + 1]);
    }
    const size_t o = static_cast<size_t>(t) * H + c * 8;
    if (out_mode == 1) {
      uint16_t* ob = reinterpret_cast<uint16_t*>(out) + o;
#pragma unroll
      for (int i = 0; i < 8; ++i) ob[i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i]));
    } else {
      float* of = reinterpret_cast<float*>(out) + o;
#pragma unroll
      for (int i = 0; i < 8; ++i) of[i] = out_mode == 2 ? of[i] + acc[i] : acc[i];
    }
  }
}

}  // namespace pf
}  // namespace moe
