// Per-layer kernels of the routed-expert layer: the decode (GEMV) path behind
// moe_route_topk, moe_expert_forward and prerouter_predict.
//
// Weights are read once per launch with 16-byte streaming loads; each warp
// segment owns a row, its lanes stride over 16-byte chunks so a warp reads
// contiguous bytes.  Dequantisation is fused into the dot product: per group of
// 64 inputs  sum_k u_k (q_k*s + b) = s * sum_k u_k (q_k - m) + (b + m*s) * sum_k u_k
// with m = 8 (int4) or 128 (8-bit); q - m is exact in fp16 and its product with
// an fp16 activation is exact in fp32, accumulated by mixed-precision FMA.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int TB = 8;  // tokens per pass of a GEMV kernel


// ----------------------------------------------------------------------------- activation staging
// Stage tokens tok[0..nt) of u (bf16 [.][H]) into shared memory as fp16:
// natural order (8 consecutive values per uint4) or pair order (per 8-block:
// (u_j, u_{j+4}) for j = 0..3).  sum32[t][c] / sum16[t][c] are fp32 sums of the
// bf16 values over 32- / 16-element chunks (may be null).  A value fp16 cannot
// hold (|u| > 65504 or not finite) reports MOE_ERR_RANGE into err (may be null).
MOE_DEV void stage_tokens(const uint16_t* __restrict__ u, int H, const int* tok, int nt, uint4* dst,
                          float* sum32, float* sum16, bool pair_order, int* err) {
  const int n32 = H / 32;
  bool bad = false;
  for (int wi = threadIdx.x; wi < nt * n32; wi += blockDim.x) {
    const int t = wi / n32, c = wi - t * n32;
    const uint4* src = reinterpret_cast<const uint4*>(u + static_cast<size_t>(tok[t]) * H + c * 32);
    float s[2] = {0.f, 0.f};
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      const uint4 v = src[blk];
      const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
      uint16_t e[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint16_t lo = static_cast<uint16_t>(vw[i] & 0xffffu), hi = static_cast<uint16_t>(vw[i] >> 16);
        const float flo = bf16_bits_to_float(lo), fhi = bf16_bits_to_float(hi);
        bad |= !(fabsf(flo) <= kF16Max) || !(fabsf(fhi) <= kF16Max);
        s[blk >> 1] += flo;
        s[blk >> 1] += fhi;
        e[2 * i] = bf16_to_f16_bits(lo);
        e[2 * i + 1] = bf16_to_f16_bits(hi);
      }
      uint4 o;
      if (pair_order) {
        o.x = e[0] | (static_cast<uint32_t>(e[4]) << 16);
        o.y = e[1] | (static_cast<uint32_t>(e[5]) << 16);
        o.z = e[2] | (static_cast<uint32_t>(e[6]) << 16);
        o.w = e[3] | (static_cast<uint32_t>(e[7]) << 16);
      } else {
        o.x = e[0] | (static_cast<uint32_t>(e[1]) << 16);
        o.y = e[2] | (static_cast<uint32_t>(e[3]) << 16);
        o.z = e[4] | (static_cast<uint32_t>(e[5]) << 16);
        o.w = e[6] | (static_cast<uint32_t>(e[7]) << 16);
      }
      dst[static_cast<size_t>(t) * (H / 8) + c * 4 + blk] = o;
    }
    if (sum32) sum32[t * n32 + c] = s[0] + s[1];
    if (sum16) {
      sum16[t * 2 * n32 + 2 * c] = s[0];
      sum16[t * 2 * n32 + 2 * c + 1] = s[1];
    }
  }
  if (bad) report(err, 6);
}


// ----------------------------------------------------------------------------- glue: RMSNorm -> bf16
__global__ void __launch_bounds__(kThreads) rmsnorm_bf16_kernel(const float* __restrict__ x, int H, float eps,
                                                                uint16_t* __restrict__ u) {
  __shared__ float red[kWarps];
  const float* xr = x + static_cast<size_t>(blockIdx.x) * H;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += kThreads) ss = fmaf(xr[i], xr[i], ss);
  ss = warp_reduce(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) tot += red[w];
  const float rs = rsqrtf(tot / static_cast<float>(H) + eps);
  uint16_t* ur = u + static_cast<size_t>(blockIdx.x) * H;
  for (int i = threadIdx.x; i < H; i += kThreads) ur[i] = __bfloat16_as_ushort(__float2bfloat16_rn(xr[i] * rs));
}

// ----------------------------------------------------------------------------- 8-bit GEMV rows
// acc[t] += row . u[t] for one 8-bit row handled by a segment of SEG lanes.
template <int NCH, int SEG>
MOE_DEV void row_int8(const uint32_t* __restrict__ q, const uint16_t* __restrict__ sc, const uint16_t* __restrict__ bi,
                      const uint4* us, const float* sum16, int nt, int sl, float (&acc)[TB]) {
  constexpr int CPL = NCH / SEG;  // 16-byte chunks per lane
  constexpr int H = NCH * 16;
  uint4 w[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) w[c] = ldg_stream(reinterpret_cast<const uint4*>(q) + sl + c * SEG);
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    const int ch = sl + c * SEG, g = ch >> 2;
    const float s = half_bits_to_float(sc[g]);
    const float b = half_bits_to_float(bi[g]) + 128.0f * s;
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      if (t < nt) {
        const float d = dot_chunk_int8(w[c], us + t * (H / 8) + ch * 2, 0.f);
        acc[t] = fmaf(s, d, fmaf(b, sum16[t * NCH + ch], acc[t]));
      }
    }
  }
}

// Router logits: logits[t][e] = W_r[e] . u[t] + bias[e].  grid (ceil(E / rows per CTA), ceil(T / TB)).
template <int NCH>  // H / 16
__global__ void __launch_bounds__(kThreads) router_kernel(const uint16_t* __restrict__ u, int T,
                                                          const uint8_t* __restrict__ rows, const float* __restrict__ rbias,
                                                          int E, float* __restrict__ logits, int* err) {
  constexpr int SEG = NCH < 32 ? NCH : 32;
  constexpr int RPW = 32 / SEG;
  constexpr int H = NCH * 16;
  constexpr int R = qrow_bytes(H, 8);
  extern __shared__ uint4 smem[];
  uint4* us = smem;
  float* sum16 = reinterpret_cast<float*>(us + TB * (H / 8));
  __shared__ int tok[TB];
  const int t0 = blockIdx.y * TB, nt = min(TB, T - t0);
  if (threadIdx.x < TB) tok[threadIdx.x] = t0 + min(static_cast<int>(threadIdx.x), nt - 1);
  __syncthreads();
  stage_tokens(u, H, tok, nt, us, nullptr, sum16, false, blockIdx.x == 0 ? err : nullptr);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sl = lane % SEG;
  const int e = (blockIdx.x * kWarps + warp) * RPW + lane / SEG;
  float acc[TB];
#pragma unroll
  for (int t = 0; t < TB; ++t) acc[t] = 0.f;
  if (e < E) {
    const uint8_t* rec = rows + static_cast<size_t>(e) * R;
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + H);
    row_int8<NCH, SEG>(reinterpret_cast<const uint32_t*>(rec), sc, sc + H / 64, us, sum16, nt, sl, acc);
  }
#pragma unroll
  for (int t = 0; t < TB; ++t) acc[t] = seg_reduce<SEG>(acc[t]);
  if (e < E && sl == 0) {
    const float rb = rbias ? rbias[e] : 0.f;
    for (int t = 0; t < nt; ++t) logits[static_cast<size_t>(t0 + t) * E + e] = acc[t] + rb;
  }
}

// ----------------------------------------------------------------------------- top-K + softmax over the K
// One warp per token.  Selects the K largest scores (descending; equal scores
// -> lower index).  w (optional): softmax of the selected scores.
__global__ void __launch_bounds__(kThreads) topk_kernel(const float* __restrict__ scores, int T, int E, int K,
                                                        int32_t* __restrict__ idx, float* __restrict__ w) {
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  constexpr int VPL = 8;  // E <= 256
  float v[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int i = lane + 32 * j;
    const float x = i < E ? scores[static_cast<size_t>(t) * E + i] : -INFINITY;
    v[j] = x == x ? x : -INFINITY;  // NaN ranks below every number
  }
  uint32_t taken = 0;
  float selv[8];
  int seli[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (k < K) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int i = lane + 32 * j;
        if (i < E && !((taken >> j) & 1u) && (v[j] > bv || (v[j] == bv && i < bi))) {
          bv = v[j];
          bi = i;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      selv[k] = bv;
      seli[k] = bi;
      if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    }
  }
  if (lane == 0) {
    float ex[8], sum = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k < K) {
        ex[k] = expf(selv[k] - selv[0]);
        sum += ex[k];
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k < K) {
        idx[static_cast<size_t>(t) * K + k] = seli[k];
        if (w) w[static_cast<size_t>(t) * K + k] = __fdividef(ex[k], sum);
      }
    }
  }
}

// Gating at given indices (predicted routing): w[t][k] = softmax over k of
// logits[t][idx[t][k]].  One warp per token; indices are clamped into [0, E).
__global__ void __launch_bounds__(kThreads) gate_at_kernel(const float* __restrict__ logits, int T, int E, int K,
                                                           const int32_t* __restrict__ idx, float* __restrict__ w) {
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (t >= T || (threadIdx.x & 31) != 0) return;
  float l[8], ex[8], sum = 0.f;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    int e = idx[static_cast<size_t>(t) * K + k];
    e = e < 0 ? 0 : (e >= E ? E - 1 : e);
    l[k] = logits[static_cast<size_t>(t) * E + e];
  }
  float m = l[0];
#pragma unroll 1
  for (int k = 1; k < K; ++k) m = fmaxf(m, l[k]);
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    ex[k] = expf(l[k] - m);
    sum += ex[k];
  }
  const float inv = __fdividef(1.0f, sum);
#pragma unroll 1
  for (int k = 0; k < K; ++k) w[static_cast<size_t>(t) * K + k] = ex[k] * inv;
}

// ----------------------------------------------------------------------------- buckets
// Single-CTA stable counting sort of the T*K slots by expert:
// count[e], offset[e] (exclusive scan, offset[E] = T*K), perm[pos] = slot,
// inv[slot] = pos.  Deterministic (no order-dependent atomics).
MOE_DEV void bucket_slots(const int32_t* __restrict__ idx, int TK, int E, int32_t* count, int32_t* offset,
                          int32_t* perm, int32_t* inv, int32_t* perm_out) {
  __shared__ int cnt[256];
  __shared__ int base[256];
  __shared__ int wcnt[kWarps][256];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int s = threadIdx.x; s < TK; s += blockDim.x) atomicAdd(&cnt[idx[s]], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      base[e] = run;
      offset[e] = run;
      count[e] = cnt[e];
      run += cnt[e];
    }
    offset[E] = run;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int c0 = 0; c0 < TK; c0 += kThreads) {
    for (int i = threadIdx.x; i < kWarps * E; i += kThreads) (&wcnt[0][0])[(i / E) * 256 + (i % E)] = 0;
    __syncthreads();
    const int s = c0 + threadIdx.x;
    const bool act = s < TK;
    const int e = act ? idx[s] : -1 - lane;  // inactive lanes never match each other
    const unsigned m = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(m & ((1u << lane) - 1u));
    if (act && rank_w == 0) wcnt[warp][e] = __popc(m);
    __syncthreads();
    if (act) {
      int pos = base[e] + rank_w;
      for (int w2 = 0; w2 < warp; ++w2) pos += wcnt[w2][e];
      perm[pos] = s;
      if (perm_out) perm_out[pos] = s;
      if (inv) inv[s] = pos;
    }
    __syncthreads();
    for (int ee = threadIdx.x; ee < E; ee += kThreads) {
      int add = 0;
      for (int w2 = 0; w2 < kWarps; ++w2) add += wcnt[w2][ee];
      base[ee] += add;
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------- fp16 GEMV rows (LoRA A, Prerouter)
// acc[t] += row . u[t] for an fp16 row of NCH 8-element chunks, natural-order u.
template <int NCH, int SEG>
MOE_DEV void row_f16(const uint16_t* __restrict__ wrow, const uint4* us, int ustride, int nt, int sl,
                     float (&acc)[TB]) {
  constexpr int CPL = NCH / SEG;
  uint4 w[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) w[c] = ldg_stream(reinterpret_cast<const uint4*>(wrow) + sl + c * SEG);
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
#pragma unroll
    for (int t = 0; t < TB; ++t)
      if (t < nt) acc[t] = dot_chunk_f16(w[c], us[t * ustride + sl + c * SEG], acc[t]);
  }
}

struct PreArgs {
  const uint16_t* u;
  int T, K, E, r;
  const int32_t* idx_in;  // caller's indices
  int32_t* idx;           // clamped copy used by every later kernel
  int32_t *count, *offset, *perm, *inv, *perm_out;
  const uint8_t* sg_rec;   // shared-gate row record (8-bit, H inputs)
  const uint16_t* A_gate;  // [r][H] or null
  const uint16_t* A_up;
  float* g;     // [T]
  float* t_gu;  // [T][2][r]
  int* err;     // optional error word
};

// Block 0: buckets.  Blocks >= 1: shared-expert gate and the shared LoRA A u
// products (gate, up), one row per warp, tokens in passes of TB.
template <int NCH8>  // H / 8
__global__ void __launch_bounds__(kThreads) pre_kernel(PreArgs a) {
  constexpr int H = NCH8 * 8;
  if (blockIdx.x == 0) {
    // indices outside [0, E) are clamped so that no kernel reads outside the pool
    for (int s = threadIdx.x; s < a.T * a.K; s += blockDim.x) {
      const int v = a.idx_in[s];
      a.idx[s] = v < 0 ? 0 : (v >= a.E ? a.E - 1 : v);
    }
    __syncthreads();
    bucket_slots(a.idx, a.T * a.K, a.E, a.count, a.offset, a.perm, a.inv, a.perm_out);
    return;
  }
  extern __shared__ uint4 smem[];
  uint4* us = smem;
  float* sum16 = reinterpret_cast<float*>(us + TB * (H / 8));
  __shared__ int tok[TB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = (blockIdx.x - 1) * kWarps + warp;  // 0: gate, 1..r: A_gate, r+1..2r: A_up
  const int nrows = 1 + (a.A_gate ? a.r : 0) + (a.A_up ? a.r : 0);
  for (int t0 = 0; t0 < a.T; t0 += TB) {
    const int nt = min(TB, a.T - t0);
    __syncthreads();
    if (threadIdx.x < TB) tok[threadIdx.x] = t0 + min(static_cast<int>(threadIdx.x), nt - 1);
    __syncthreads();
    stage_tokens(a.u, H, tok, nt, us, nullptr, sum16, false, blockIdx.x == 1 ? a.err : nullptr);
    __syncthreads();
    float acc[TB];
#pragma unroll
    for (int t = 0; t < TB; ++t) acc[t] = 0.f;
    if (row == 0) {
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(a.sg_rec + H);
      row_int8<H / 16, 32 < H / 16 ? 32 : H / 16>(reinterpret_cast<const uint32_t*>(a.sg_rec), sc, sc + H / 64, us,
                                                   sum16, nt, lane % (32 < H / 16 ? 32 : H / 16), acc);
      constexpr int SEG = 32 < H / 16 ? 32 : H / 16;
#pragma unroll
      for (int t = 0; t < TB; ++t) acc[t] = seg_reduce<SEG>(acc[t]);
      if (lane == 0)
        for (int t = 0; t < nt; ++t) a.g[t0 + t] = sigmoid(acc[t]);
    } else if (row < nrows) {
      constexpr int SEG = NCH8 < 32 ? NCH8 : 32;
      const int i = row - 1;
      const bool is_gate = a.A_gate && i < a.r;
      const int ri = is_gate ? i : (a.A_gate ? i - a.r : i);
      const uint16_t* A = is_gate ? a.A_gate : a.A_up;
      if (lane < SEG) row_f16<NCH8, SEG>(A + static_cast<size_t>(ri) * H, us, H / 8, nt, lane, acc);
#pragma unroll
      for (int t = 0; t < TB; ++t) acc[t] = seg_reduce<32>(acc[t]);
      if (lane == 0)
        for (int t = 0; t < nt; ++t) a.t_gu[(static_cast<size_t>(t0 + t) * 2 + (is_gate ? 0 : 1)) * a.r + ri] = acc[t];
    }
  }
}

// ----------------------------------------------------------------------------- gate/up + SwiGLU
struct GateUpArgs {
  const uint16_t* u;
  int T, K, I;
  const int32_t *idx, *perm, *offset;
  const uint8_t* pool;
  int64_t stride;
  const uint8_t* sh_block;        // shared expert block
  const uint16_t *sh_Bg, *sh_Bu;  // [I][r] or null
  const float* t_gu;              // [T][2][r]
  int r;
  float lora_scale;
  uint16_t* h16;  // [T*K + T][I] fp16, pair order
  int* err;       // optional error word: a SwiGLU output fp16 cannot hold reports MOE_ERR_RANGE
};

// grid (ceil(I / pairs per CTA), T*K + 1).  Unit y < T*K is the sorted slot
// position y; it works only when it starts its expert's bucket and then covers
// the whole bucket.  Unit T*K is the shared expert over all T tokens.
template <int NCH>  // H / 32
__global__ void __launch_bounds__(kThreads) gate_up_kernel(GateUpArgs a) {
  constexpr int SEG = NCH < 32 ? NCH : 32;
  constexpr int CPL = NCH / SEG;
  constexpr int PPW = 32 / SEG;
  constexpr int H = NCH * 32;
  constexpr int G = H / 64;
  constexpr int RGU = qrow_bytes(H, 4);
  extern __shared__ uint4 smem[];
  uint4* up = smem;
  float* sum32 = reinterpret_cast<float*>(up + TB * (H / 8));
  __shared__ int tok[TB];
  __shared__ int slot[TB];
  const int TK = a.T * a.K;
  const int unit = blockIdx.y;
  const bool shared = unit == TK;
  int start = 0, n = a.T;
  const uint8_t* blk = a.sh_block;
  if (!shared) {
    const int e = a.idx[a.perm[unit]];
    if (a.offset[e] != unit) return;
    start = unit;
    n = a.offset[e + 1] - unit;
    blk = a.pool + static_cast<int64_t>(e) * a.stride;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sl = lane % SEG;
  const int j = (blockIdx.x * kWarps + warp) * PPW + lane / SEG;
  if (blockIdx.x * kWarps * PPW >= a.I) return;
  const bool valid = j < a.I;
  for (int p0 = 0; p0 < n; p0 += TB) {
    const int nt = min(TB, n - p0);
    __syncthreads();
    if (threadIdx.x < TB) {
      const int i = min(static_cast<int>(threadIdx.x), nt - 1);
      const int s = shared ? TK + p0 + i : a.perm[start + p0 + i];
      slot[threadIdx.x] = s;
      tok[threadIdx.x] = shared ? p0 + i : s / a.K;
    }
    __syncthreads();
    stage_tokens(a.u, H, tok, nt, up, sum32, nullptr, true, nullptr);
    __syncthreads();
    float ag[TB], au[TB];
#pragma unroll
    for (int t = 0; t < TB; ++t) ag[t] = au[t] = 0.f;
    if (valid) {
      const uint8_t* rg = blk + static_cast<size_t>(2 * j) * RGU;  // gate row j, then up row j
      const uint8_t* ru = rg + RGU;
      const uint4* qg = reinterpret_cast<const uint4*>(rg);
      const uint4* qu = reinterpret_cast<const uint4*>(ru);
      const uint16_t* sgp = reinterpret_cast<const uint16_t*>(rg + H / 2);
      const uint16_t* sup = reinterpret_cast<const uint16_t*>(ru + H / 2);
      uint4 wg[CPL], wu[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        wg[c] = ldg_stream(qg + sl + c * SEG);
        wu[c] = ldg_stream(qu + sl + c * SEG);
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const int ch = sl + c * SEG, g = ch >> 1;
        const float sg = half_bits_to_float(sgp[g]);
        const float bg = half_bits_to_float(sgp[G + g]) + 8.0f * sg;
        const float su = half_bits_to_float(sup[g]);
        const float bu = half_bits_to_float(sup[G + g]) + 8.0f * su;
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          if (t < nt) {
            const uint4* ut = up + t * (H / 8) + ch * 4;
            const float us = sum32[t * NCH + ch];
            ag[t] = fmaf(sg, dot_chunk_int4(wg[c], ut, 0.f), fmaf(bg, us, ag[t]));
            au[t] = fmaf(su, dot_chunk_int4(wu[c], ut, 0.f), fmaf(bu, us, au[t]));
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      ag[t] = seg_reduce<SEG>(ag[t]);
      au[t] = seg_reduce<SEG>(au[t]);
    }
    if (valid && sl == 0) {
      for (int t = 0; t < nt; ++t) {
        float gv = ag[t], uv = au[t];
        if (shared) {
          const float* tg = a.t_gu + static_cast<size_t>(tok[t]) * 2 * a.r;
          if (a.sh_Bg) {
            float d = 0.f;
            for (int i = 0; i < a.r; ++i) d = fmaf(half_bits_to_float(a.sh_Bg[static_cast<size_t>(j) * a.r + i]), tg[i], d);
            gv = fmaf(a.lora_scale, d, gv);
          }
          if (a.sh_Bu) {
            float d = 0.f;
            for (int i = 0; i < a.r; ++i)
              d = fmaf(half_bits_to_float(a.sh_Bu[static_cast<size_t>(j) * a.r + i]), tg[a.r + i], d);
            uv = fmaf(a.lora_scale, d, uv);
          }
        }
        const float h = silu(gv) * uv;
        if (!(fabsf(h) <= kF16Max)) report(a.err, 6);
        a.h16[static_cast<size_t>(slot[t]) * a.I + pair_pos(j)] = __half_as_ushort(__float2half_rn(h));
      }
    }
  }
}

// ----------------------------------------------------------------------------- LoRA A h (after gate/up)
// t_ds[t][i] = A_down_shared[i] . h_shared[t];  t_ex[slot][i] = A_e[i] . h[slot] (routed down LoRA).
// One warp per (vector, i); h is fp16 in pair order, A rows fp16 natural order.
struct MidArgs {
  int T, K, I, r;
  const int32_t* idx;
  const uint16_t* h16;
  const uint16_t* A_sd;  // [r][I] or null
  const uint16_t* A_ex;  // [E][r][I] or null
  float* t_ds;           // [T][r]
  float* t_ex;           // [T*K][r]
};

__global__ void __launch_bounds__(kThreads) lora_mid_kernel(MidArgs a) {
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int TK = a.T * a.K;
  const int n_sh = a.A_sd ? a.T * a.r : 0;
  const int n_ex = a.A_ex ? TK * a.r : 0;
  if (gw >= n_sh + n_ex) return;
  const uint16_t* A;
  const uint16_t* h;
  float* dst;
  if (gw < n_sh) {
    const int t = gw / a.r, i = gw % a.r;
    A = a.A_sd + static_cast<size_t>(i) * a.I;
    h = a.h16 + static_cast<size_t>(TK + t) * a.I;
    dst = a.t_ds + gw;
  } else {
    const int x = gw - n_sh, s = x / a.r, i = x % a.r;
    A = a.A_ex + (static_cast<size_t>(a.idx[s]) * a.r + i) * a.I;
    h = a.h16 + static_cast<size_t>(s) * a.I;
    dst = a.t_ex + x;
  }
  float acc = 0.f;
  for (int c = lane; c < a.I / 8; c += 32) {
    const uint4 w = *reinterpret_cast<const uint4*>(A + c * 8);
    const uint4 hv = *reinterpret_cast<const uint4*>(h + c * 8);
    // A chunk in natural order -> pair order, to match h
    const uint32_t p0 = prmt(w.x, w.z, 0x5410u), p1 = prmt(w.x, w.z, 0x7632u);
    const uint32_t p2 = prmt(w.y, w.w, 0x5410u), p3 = prmt(w.y, w.w, 0x7632u);
    acc = dot2_mix(p0, hv.x, acc);
    acc = dot2_mix(p1, hv.y, acc);
    acc = dot2_mix(p2, hv.z, acc);
    acc = dot2_mix(p3, hv.w, acc);
  }
  acc = warp_reduce(acc);
  if (lane == 0) *dst = acc;
}

// ----------------------------------------------------------------------------- down + combine
struct DownArgs {
  int T, K, H, I, r;
  const int32_t* idx;
  const float* w;
  const float* g;
  const uint8_t* pool;
  int64_t stride;
  const uint8_t* sh_block;
  const uint16_t* B_sd;  // [H][r] or null
  const uint16_t* B_ex;  // [E][H][r] or null
  const float* t_ds;
  const float* t_ex;
  float lora_scale;
  const uint16_t* h16;
  void* out;
  int out_mode;
};

// One warp per output row o; per token, the K routed down rows and the shared
// down row are processed SPP at a time (SEG lanes each), then combined by lane
// 0 in fixed order: sum_k w_k y_k, then + g y_shared.
template <int NCH>  // I / 32
__global__ void __launch_bounds__(kThreads) down_kernel(DownArgs a) {
  constexpr int SEG = NCH < 32 ? NCH : 32;
  constexpr int CPL = NCH / SEG;
  constexpr int SPP = 32 / SEG;
  constexpr int I = NCH * 32;
  constexpr int G = I / 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sl = lane % SEG, sub = lane / SEG;
  const int o = blockIdx.x * kWarps + warp;
  if (o >= a.H) return;
  constexpr int RDN = qrow_bytes(I, 4);
  const size_t dn_off = static_cast<size_t>(2 * I) * qrow_bytes(a.H, 4) + static_cast<size_t>(o) * RDN;
  const int TK = a.T * a.K;
  for (int t = 0; t < a.T; ++t) {
    float acc = 0.f;
    for (int p0 = 0; p0 <= a.K; p0 += SPP) {
      const int k = p0 + sub;
      float y = 0.f;
      int e = -1;
      if (k <= a.K) {
        const uint8_t* rec;
        const uint16_t* h;
        if (k < a.K) {
          e = a.idx[t * a.K + k];
          rec = a.pool + static_cast<int64_t>(e) * a.stride + dn_off;
          h = a.h16 + static_cast<size_t>(t * a.K + k) * I;
        } else {
          rec = a.sh_block + dn_off;
          h = a.h16 + static_cast<size_t>(TK + t) * I;
        }
        const uint32_t* q = reinterpret_cast<const uint32_t*>(rec);
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + I / 2);
        const uint16_t* bi = sc + G;
        uint4 wv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) wv[c] = ldg_stream(reinterpret_cast<const uint4*>(q) + sl + c * SEG);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const int ch = sl + c * SEG, g = ch >> 1;
          const float s = half_bits_to_float(sc[g]);
          const float b = half_bits_to_float(bi[g]) + 8.0f * s;
          const uint4* hp = reinterpret_cast<const uint4*>(h) + ch * 4;
          uint4 hv[4];
          float hs = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            hv[i] = hp[i];
            const uint32_t hw[4] = {hv[i].x, hv[i].y, hv[i].z, hv[i].w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float2 f = __half22float2(as_h2(hw[m]));
              hs += f.x + f.y;
            }
          }
          y = fmaf(s, dot_chunk_int4(wv[c], hv, 0.f), fmaf(b, hs, y));
        }
      }
      y = seg_reduce<SEG>(y);
      if (sl == 0 && k <= a.K) {
        if (k < a.K && a.B_ex) {
          const uint16_t* B = a.B_ex + (static_cast<size_t>(e) * a.H + o) * a.r;
          const float* tv = a.t_ex + static_cast<size_t>(t * a.K + k) * a.r;
          float d = 0.f;
          for (int i = 0; i < a.r; ++i) d = fmaf(half_bits_to_float(B[i]), tv[i], d);
          y = fmaf(a.lora_scale, d, y);
        } else if (k == a.K && a.B_sd) {
          const uint16_t* B = a.B_sd + static_cast<size_t>(o) * a.r;
          const float* tv = a.t_ds + static_cast<size_t>(t) * a.r;
          float d = 0.f;
          for (int i = 0; i < a.r; ++i) d = fmaf(half_bits_to_float(B[i]), tv[i], d);
          y = fmaf(a.lora_scale, d, y);
        }
      }
#pragma unroll
      for (int s2 = 0; s2 < SPP; ++s2) {
        const float v = __shfl_sync(0xffffffffu, y, s2 * SEG);
        const int kk = p0 + s2;
        if (lane == 0) {
          if (kk < a.K) acc = fmaf(a.w[t * a.K + kk], v, acc);
          else if (kk == a.K) acc = fmaf(a.g[t], v, acc);
        }
      }
    }
    if (lane == 0) {
      const size_t oi = static_cast<size_t>(t) * a.H + o;
      if (a.out_mode == 0) reinterpret_cast<float*>(a.out)[oi] = acc;
      else if (a.out_mode == 1) reinterpret_cast<uint16_t*>(a.out)[oi] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
      else reinterpret_cast<float*>(a.out)[oi] += acc;
    }
  }
}

// ----------------------------------------------------------------------------- Prerouter
struct PreW1Args {
  const uint16_t* u;
  int T, K, E, P;
  const int32_t* sel;
  const uint16_t *W1, *b1;
  float* z;  // [T][P]
  int* err;  // optional error word
};

// z[t][p] = silu(W1[p][:H] . u[t] + sum_k W1[p][H + sel[t][k]] + b1[p]); one row per warp.
template <int NCH8>  // H / 8
__global__ void __launch_bounds__(kThreads) prerouter_w1_kernel(PreW1Args a) {
  constexpr int H = NCH8 * 8;
  constexpr int SEG = NCH8 < 32 ? NCH8 : 32;
  extern __shared__ uint4 smem[];
  uint4* us = smem;
  __shared__ int tok[TB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x * kWarps + warp;
  const int t0 = blockIdx.y * TB, nt = min(TB, a.T - t0);
  if (threadIdx.x < TB) tok[threadIdx.x] = t0 + min(static_cast<int>(threadIdx.x), nt - 1);
  __syncthreads();
  stage_tokens(a.u, H, tok, nt, us, nullptr, nullptr, false, blockIdx.x == 0 ? a.err : nullptr);
  __syncthreads();
  if (p >= a.P) return;
  float acc[TB];
#pragma unroll
  for (int t = 0; t < TB; ++t) acc[t] = 0.f;
  const uint16_t* row = a.W1 + static_cast<size_t>(p) * (H + a.E);
  if (lane < SEG) row_f16<NCH8, SEG>(row, us, H / 8, nt, lane, acc);
#pragma unroll
  for (int t = 0; t < TB; ++t) acc[t] = seg_reduce<32>(acc[t]);
  if (lane == 0) {
    const float b = half_bits_to_float(a.b1[p]);
    for (int t = 0; t < nt; ++t) {
      float m = 0.f;
      for (int k = 0; k < a.K; ++k) {
        int e = a.sel[static_cast<size_t>(t0 + t) * a.K + k];
        e = e < 0 ? 0 : (e >= a.E ? a.E - 1 : e);  // out-of-range selections are clamped
        m += half_bits_to_float(row[H + e]);
      }
      a.z[static_cast<size_t>(t0 + t) * a.P + p] = silu(acc[t] + m + b);
    }
  }
}

// Second Prerouter layer: scores[t][e] = b2[e] + sum_p W2[e][p] * z[t][p], register-tiled.  A CTA of 256
// threads takes 64 tokens x 64 rows, each thread 4 tokens x 4 rows; z and W2 (as fp32) are staged in shared
// memory 32 inputs at a time, input-major, so a thread reads one float4 of each per input.  A chunk's 32
// products are summed in order and the chunk sum is added to the total: at most 32 + ceil(P/32) + 1 fp32
// roundings on the path of any product.
constexpr int kW2T = 64, kW2E = 64, kW2K = 32, kW2Threads = 256;
__global__ void __launch_bounds__(kW2Threads) prerouter_w2_kernel(const float* __restrict__ z, int T, int P,
                                                                   const uint16_t* __restrict__ W2,
                                                                   const uint16_t* __restrict__ b2, int En,
                                                                   float* __restrict__ scores) {
  __shared__ __align__(16) float zs[kW2K][kW2T + 4];
  __shared__ __align__(16) float ws[kW2K][kW2E + 4];
  const int t0 = blockIdx.y * kW2T, e0 = blockIdx.x * kW2E;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // rows e0 + 4 tx + j, tokens t0 + 4 ty + i
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 1
  for (int p0 = 0; p0 < P; p0 += kW2K) {
    const int pc = min(kW2K, P - p0);
    __syncthreads();
    for (int i = threadIdx.x; i < kW2T * kW2K; i += kW2Threads) {
      const int tt = i / kW2K, pp = i % kW2K, t = t0 + tt;  // consecutive threads: consecutive inputs
      zs[pp][tt] = (t < T && pp < pc) ? z[static_cast<size_t>(t) * P + p0 + pp] : 0.f;
    }
    for (int i = threadIdx.x; i < kW2E * kW2K; i += kW2Threads) {
      const int ee = i / kW2K, pp = i % kW2K, e = e0 + ee;
      ws[pp][ee] = (e < En && pp < pc) ? half_bits_to_float(W2[static_cast<size_t>(e) * P + p0 + pp]) : 0.f;
    }
    __syncthreads();
    float part[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
#pragma unroll 8
    for (int pp = 0; pp < kW2K; ++pp) {
      const float4 zv = *reinterpret_cast<const float4*>(&zs[pp][4 * ty]);
      const float4 wv = *reinterpret_cast<const float4*>(&ws[pp][4 * tx]);
      const float zz[4] = {zv.x, zv.y, zv.z, zv.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(zz[i], ww[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = e0 + 4 * tx + j;
    if (e >= En) continue;
    const float b = half_bits_to_float(b2[e]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + 4 * ty + i;
      if (t < T) scores[static_cast<size_t>(t) * En + e] = acc[i][j] + b;
    }
  }
}

}  // namespace moe
