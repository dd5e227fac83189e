// Persistent fused decode of a whole MoE stack for one token (batch 1), second
// generation: the same work split as the first single-launch kernel, with the
// per-layer critical path rearranged so that no phase runs on one warp while
// the others wait, and so that the waits on the three all-to-all exchanges are
// filled with work that does not depend on them.
//
// Per layer, each CTA (one per SM, 512 threads):
//  A  x received -> RMSNorm -> u; its router / shared-gate / LoRA-A rows
//     (8-bit and fp16 GEMV rows) -> published as epoch words;
//     then, while the logits travel: the shared expert's (gate, up) dot products
//     and the Prerouter's hidden rows on u (both token-independent weights,
//     prefetched one layer ahead into shared memory);
//  B  logits received -> every warp selects the top-K itself (the same
//     deterministic result, no block barrier) -> each warp issues its share of
//     the routed-row bulk copies -> shared pairs get their LoRA delta, routed
//     pairs are computed as their rows land -> SwiGLU outputs and Prerouter
//     hidden values published;
//  C  hidden vector received (straight into pair order, with its 32-value chunk
//     sums) -> down rows of the K routed experts and the shared expert -> combine
//     (16 lanes per output row) -> x rows published.
// The Prerouter heads' output layers and predictions are off the per-layer
// path: every layer publishes its hidden values z, and after the last layer
// each CTA computes its output rows of every head and the CTAs split the
// predictions.
// Exchanges use 64-bit epoch words (32-bit payload, 32-bit layer epoch;
// single-copy-atomic stores and loads), every thread spinning on its own share.
// Every wait is bounded by %globaltimer; on timeout the CTA records
// MOE_ERR_TIMEOUT, waits (bounded) for its own bulk copies and returns.
#pragma once

#include "stack_kernel.cuh"

namespace moe {
namespace stk2 {

using stk::bulk_load;
using stk::fence_proxy_async;
using stk::gtimer;
using stk::key_value;
using stk::kMaxLayers;
using stk::kTraceSlots;
using stk::LayerPtrs;
using stk::ld_word;
using stk::mbar_expect;
using stk::mbar_init;
using stk::mbar_wait;
using stk::ord_key;
using stk::split;
using stk::st_word;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxK = 8;

// Byte offsets into dynamic shared memory (computed on the host).
struct Smem {
  uint32_t st[2];                                           // static (token-independent) buffers
  uint32_t o_items, o_shu, o_shB, o_sdn, o_Bd, o_Ad, o_W1;  // offsets inside a static buffer
  uint32_t units, down;                                     // routed rows
  uint32_t xs, un, up, s16, s32, hs, hsum, logit, td, yd, red, zx, hloc, shacc, bar;
  uint32_t total;
  int maxA, maxS, maxR, maxD, maxZ, item_bytes;
};

struct Params {
  int n_layers, E, K, r, P, En, NA;
  int64_t stride;
  float eps, lora_scale;
  float* x;
  float* x_trace;
  uint16_t* u_trace;
  int32_t* idx_all;
  int32_t* true_idx_all;
  int32_t* pred_all;
  int32_t* err;
  unsigned long long* ll;  // epoch words, zeroed before the launch
  int ll_x, ll_a, ll_h, ll_stride;  // per-parity regions (x, router items, SwiGLU outputs)
  int ll_z, ll_p;                   // per layer: Prerouter hidden values at ll_z + l*P, scores at ll_p + l*En
  int st_bytes;                     // bytes of one static buffer (scratch for the Prerouter tail)
  long long timeout_ns;
  int drop_layer, drop_cta;  // test hook: that CTA never publishes its residual rows of that layer
  long long* trace;          // optional [n_layers][grid][kTraceSlots] globaltimer stamps
  Smem sm;
  LayerPtrs L[kMaxLayers];
};

// Every thread waits for its share of the n epoch words of `epoch` (spinning on
// each word in turn) and stores the payloads to dst.  Block-uniform false on timeout.
__device__ __noinline__ bool gather(const unsigned long long* buf, int n, uint32_t epoch, long long timeout_ns,
                                    uint32_t* dst) {
  const long long deadline = gtimer() + timeout_ns;
  int bad = 0;
#pragma unroll 1
  for (int i = threadIdx.x; i < n && !bad; i += blockDim.x) {
    unsigned long long v = ld_word(buf + i);
#pragma unroll 1
    for (int it = 1; static_cast<uint32_t>(v >> 32) != epoch; ++it) {
      if ((it & 15) == 0 && gtimer() > deadline) {
        bad = 1;
        break;
      }
      v = ld_word(buf + i);
    }
    dst[i] = static_cast<uint32_t>(v);
  }
  return !__syncthreads_or(bad);
}

// Top-K of E <= 256 scores in shared memory by one warp: lane k < K returns the
// k-th expert (descending score, equal scores -> lower index) in e_out and its
// softmax weight over the K in w_out.  Every warp may run it on the same scores
// and gets the same answer.  on_slot(k, e) runs (warp-wide) as soon as slot k
// is decided.
struct NoSlot {
  MOE_DEV void operator()(int, int) const {}
};

template <typename OnSlot>
__device__ __noinline__ void warp_select(const float* sc, int E, int K, int& e_out, float& w_out, const OnSlot& on_slot) {
  const int lane = threadIdx.x & 31;
  uint32_t key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = lane + 32 * j;
    float v = i < E ? sc[i] : -INFINITY;
    if (v != v) v = -INFINITY;           // NaN ranks with -inf
    key[j] = i < E ? ord_key(v) : 0u;    // 0 is below every real key
  }
  uint32_t bk = 0u;
  int bj = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (key[j] > bk) {  // strict: the lowest j wins among equal keys of this lane
      bk = key[j];
      bj = j;
    }
  int e_sel = 0;
  uint32_t k_sel = 0u;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t win = __reduce_min_sync(0xffffffffu, bk == m ? static_cast<uint32_t>(lane + 32 * bj) : 0xffffffffu);
    const int e = static_cast<int>(win) < E ? static_cast<int>(win) : 0;
    if (lane == k) {
      e_sel = e;
      k_sel = m;
    }
    if (static_cast<int>(win & 31u) == lane) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j == static_cast<int>(win >> 5)) key[j] = 0u;
      bk = 0u;
      bj = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (key[j] > bk) {
          bk = key[j];
          bj = j;
        }
    }
    on_slot(k, e);
  }
  // softmax over the K selected values: lane k holds exp(l_k - l_0); the sum is taken in k order
  const float l0 = __shfl_sync(0xffffffffu, key_value(k_sel), 0);
  const float ex = lane < K ? expf(key_value(k_sel) - l0) : 0.f;
  float sum = 0.f;
#pragma unroll 1
  for (int k = 0; k < K; ++k) sum += __shfl_sync(0xffffffffu, ex, k);
  e_out = e_sel;
  w_out = ex * __fdividef(1.0f, sum);
}

// The routed-row copies of a CTA: copy j is its unit r0 + j for j < nR, else the
// down-row block of slot j - nR.
struct RoutedCopies {
  const uint8_t* pool;
  int64_t stride;
  uint8_t* units;
  uint8_t* down;
  uint64_t* bar_unit;
  uint64_t* bar_down;
  int r0, nR, ncopy, d0, nD, maxD, half_i, rgu, rdn, unit, i2;
  MOE_DEV int slot(int j) const { return j < nR ? (r0 + j) / half_i : j - nR; }
  // Copy j of expert e, issued by lane 0 of the calling warp with its mbarrier armed.
  MOE_DEV void issue(int j, int e) const {
    if ((threadIdx.x & 31) != 0) return;
    const int k = slot(j);
    const uint8_t* blk = pool + static_cast<int64_t>(e) * stride;
    fence_proxy_async();
    if (j < nR) {
      const int uu = r0 + j - k * half_i;
      mbar_expect(bar_unit + j, unit);
      bulk_load(units + j * unit, blk + static_cast<size_t>(4 * uu) * rgu, unit, bar_unit + j);
    } else {
      mbar_expect(bar_down + k, static_cast<uint32_t>(nD * rdn));
      bulk_load(down + (k * maxD) * rdn, blk + static_cast<size_t>(i2) * rgu + static_cast<size_t>(d0) * rdn,
                nD * rdn, bar_down + k);
    }
  }
};

// The SwiGLU outputs of all K+1 slots: every thread waits for its share of the
// (K+1)*I/2 epoch words (two fp16 values each), stores them in pair order to hs
// and, per 16 words (32 values), their fp32 sum to hsum.  n is a multiple of 32.
// Block-uniform false on timeout.
__device__ __noinline__ bool gather_h(const unsigned long long* buf, int n, int half_i, uint32_t epoch,
                                      long long timeout_ns, uint16_t* hs, float* hsum) {
  const long long deadline = gtimer() + timeout_ns;
  const int I = 2 * half_i;
  int bad = 0;
#pragma unroll 1
  for (int w = threadIdx.x; w < n; w += blockDim.x) {  // whole warps: n and blockDim are multiples of 32
    unsigned long long v = ld_word(buf + w);
#pragma unroll 1
    for (int it = 1; !bad && static_cast<uint32_t>(v >> 32) != epoch; ++it) {
      if ((it & 15) == 0 && gtimer() > deadline) bad = 1;
      v = ld_word(buf + w);
    }
    const int k = w / half_i, j = 2 * (w - k * half_i);
    const uint16_t lo = static_cast<uint16_t>(v & 0xffffu), hi = static_cast<uint16_t>((v >> 16) & 0xffffu);
    hs[k * I + pair_pos(j)] = lo;
    hs[k * I + pair_pos(j + 1)] = hi;
    float t = half_bits_to_float(lo) + half_bits_to_float(hi);
    t = seg_reduce<16>(t);
    if ((threadIdx.x & 15) == 0) hsum[w >> 4] = t;
  }
  return !__syncthreads_or(bad);
}

// Issue the token-independent weights of layer l into static buffer b (one warp;
// one bulk copy per lane per task).
template <int H, int I>
__device__ __noinline__ void issue_static(const Params& p, uint8_t* sm, uint64_t* bar, int l, int b, int s0, int s1,
                                          int d0, int d1, int z0, int z1) {
  constexpr int RGU = qrow_bytes(H, 4), RDN = qrow_bytes(I, 4), R8 = qrow_bytes(H, 8), UNIT = 4 * RGU;
  const Smem& S = p.sm;
  const int c = blockIdx.x, N = gridDim.x, lane = threadIdx.x & 31, E = p.E, r = p.r;
  const int nS = s1 - s0, nD = d1 - d0;
  const LayerPtrs& L = p.L[l];
  uint8_t* base = sm + S.st[b];
  uint32_t bytes = 0;
  for (int i = c; i < p.NA; i += N) bytes += i < E + 1 ? R8 : 2 * H;
  bytes += nS * UNIT + nD * RDN;
  if (L.Bg) bytes += nS * 4 * r;
  if (L.Bu) bytes += nS * 4 * r;
  if (L.Bd) bytes += nD * 2 * r + r * I * 2;
  if (L.W1) bytes += (z1 - z0) * 2 * H;
  fence_proxy_async();
  if (lane == 0) mbar_expect(bar + b, bytes);
  __syncwarp();
  int t = 0;
  auto task = [&](void* dst, const void* src, uint32_t n) {
    if (n && (t++ % 32) == lane) bulk_load(dst, src, n, bar + b);
  };
#pragma unroll 1
  for (int m = 0, i = c; i < p.NA; i += N, ++m) {  // phase-A items: router rows, shared gate, LoRA A rows
    uint8_t* dst = base + S.o_items + m * S.item_bytes;
    if (i < E) task(dst, L.router + static_cast<size_t>(i) * R8, R8);
    else if (i == E) task(dst, L.sgate, R8);
    else {
      const int a = i - E - 1;
      task(dst, a < r ? L.Ag + static_cast<size_t>(a) * H : L.Au + static_cast<size_t>(a - r) * H, 2 * H);
    }
  }
#pragma unroll 1
  for (int s = 0; s < nS; ++s) {
    task(base + S.o_shu + s * UNIT, L.shared + static_cast<size_t>(4 * (s0 + s)) * RGU, UNIT);
    if (L.Bg) task(base + S.o_shB + s * 8 * r, L.Bg + static_cast<size_t>(2 * (s0 + s)) * r, 4 * r);
    if (L.Bu) task(base + S.o_shB + s * 8 * r + 4 * r, L.Bu + static_cast<size_t>(2 * (s0 + s)) * r, 4 * r);
  }
  task(base + S.o_sdn, L.shared + static_cast<size_t>(2 * I) * RGU + static_cast<size_t>(d0) * RDN, nD * RDN);
  if (L.Bd) {
    task(base + S.o_Bd, L.Bd + static_cast<size_t>(d0) * r, nD * 2 * r);
    task(base + S.o_Ad, L.Ad, r * I * 2);
  }
  if (L.W1) {
#pragma unroll 1
    for (int z = z0; z < z1; ++z)
      task(base + S.o_W1 + (z - z0) * 2 * H, L.W1 + static_cast<size_t>(z) * (H + E), 2 * H);
  }
}

// (gate, up) dot products of one pair (rows 2q and 2q+1 of a unit record rec4)
// with u, by one warp; lane 0 holds the results.
template <int H>
MOE_DEV void pair_dots(const uint8_t* rec4, int q, const uint4* up, const float* s32, float& ag, float& au) {
  constexpr int G = H / 64;
  constexpr int RGU = qrow_bytes(H, 4);
  constexpr int CPL = (H / 32) / 32;
  const int lane = threadIdx.x & 31;
  const uint8_t* rg = rec4 + (2 * q) * RGU;
  const uint8_t* ru = rg + RGU;
  const uint16_t* sg = reinterpret_cast<const uint16_t*>(rg + H / 2);
  const uint16_t* su = reinterpret_cast<const uint16_t*>(ru + H / 2);
  float g = 0.f, u = 0.f;
#pragma unroll
  for (int cc = 0; cc < CPL; ++cc) {
    const int ch = lane + 32 * cc, gi = ch >> 1;
    const uint4 wg = reinterpret_cast<const uint4*>(rg)[ch];
    const uint4 wu = reinterpret_cast<const uint4*>(ru)[ch];
    const float us = s32[ch];
    const float sgv = half_bits_to_float(sg[gi]), sug = half_bits_to_float(su[gi]);
    g = fmaf(sgv, dot_chunk_int4(wg, up + 4 * ch, 0.f), fmaf(half_bits_to_float(sg[G + gi]) + 8.0f * sgv, us, g));
    u = fmaf(sug, dot_chunk_int4(wu, up + 4 * ch, 0.f), fmaf(half_bits_to_float(su[G + gi]) + 8.0f * sug, us, u));
  }
  ag = warp_reduce(g);
  au = warp_reduce(u);
}

// Prerouter heads after the last layer: every head's second layer and its
// prediction.  Each CTA gathers the hidden values z of all heads (published
// layer by layer; epoch = layer + 1) into zall (shared-memory scratch of
// cap floats, a chunk of heads at a time), computes its output rows [v0, v1) of
// every head and publishes them; then the CTAs c, c + N, ... each gather one
// head's scores and write its top-K to pred_all.
__device__ __noinline__ bool prerouter_tail(const Params& p, int v0, int v1, float* zall, int cap, float* scratch) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, c = blockIdx.x, N = gridDim.x;
  const int n = p.n_layers, P = p.P;
  const int per = cap / P > 0 ? cap / P : 1;
  const unsigned long long* zb = p.ll + p.ll_z;
  const long long deadline = gtimer() + p.timeout_ns;
  int bad = 0;
#pragma unroll 1
  for (int l0 = 0; l0 < n; l0 += per) {
    const int nl = n - l0 < per ? n - l0 : per;
#pragma unroll 1
    for (int i = tid; i < nl * P; i += blockDim.x) {
      const uint32_t ep = static_cast<uint32_t>(l0 + i / P + 1);
      unsigned long long v = ld_word(zb + static_cast<size_t>(l0) * P + i);
#pragma unroll 1
      for (int it = 1; !bad && static_cast<uint32_t>(v >> 32) != ep; ++it) {
        if ((it & 15) == 0 && gtimer() > deadline) bad = 1;
        v = ld_word(zb + static_cast<size_t>(l0) * P + i);
      }
      zall[i] = __uint_as_float(static_cast<uint32_t>(v));
    }
    if (__syncthreads_or(bad)) return false;
    const int nv = v1 - v0;
#pragma unroll 1
    for (int t = warp; t < nl * nv; t += kWarps) {  // one warp per (head, output row)
      const int lp = l0 + t / nv, e = v0 + t % nv;
      const LayerPtrs& L = p.L[lp];
      const uint4* w2 = reinterpret_cast<const uint4*>(L.W2 + static_cast<size_t>(e) * P);
      const float* z = zall + static_cast<size_t>(lp - l0) * P;
      float acc = 0.f;
#pragma unroll 1
      for (int ch = lane; ch < P / 8; ch += 32) {
        const uint4 w = w2[ch];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float2 f = __half22float2(as_h2(ws[m]));
          acc = fmaf(f.x, z[ch * 8 + 2 * m], acc);
          acc = fmaf(f.y, z[ch * 8 + 2 * m + 1], acc);
        }
      }
      acc = warp_reduce(acc);
      if (lane == 0)
        st_word(p.ll + p.ll_p + static_cast<size_t>(lp) * p.En + e, __float_as_uint(acc + half_bits_to_float(L.b2[e])),
                static_cast<uint32_t>(lp + 1));
    }
    __syncthreads();
  }
  // predictions: one warp per head
  if (warp == 0) {
#pragma unroll 1
    for (int lp = c; lp < n; lp += N) {
      const unsigned long long* pb = p.ll + p.ll_p + static_cast<size_t>(lp) * p.En;
#pragma unroll 1
      for (int i = lane; i < p.En; i += 32) {
        unsigned long long v = ld_word(pb + i);
#pragma unroll 1
        for (int it = 1; !bad && static_cast<uint32_t>(v >> 32) != static_cast<uint32_t>(lp + 1); ++it) {
          if ((it & 15) == 0 && gtimer() > deadline) bad = 1;
          v = ld_word(pb + i);
        }
        scratch[i] = __uint_as_float(static_cast<uint32_t>(v));
      }
      if (__any_sync(0xffffffffu, bad)) break;
      __syncwarp();
      int e;
      float w;
      warp_select(scratch, p.En, p.K, e, w, NoSlot{});
      if (lane < p.K && p.pred_all) p.pred_all[static_cast<size_t>(lp) * p.K + lane] = e;
      __syncwarp();
    }
  }
  return !__syncthreads_or(bad);
}

// ----------------------------------------------------------------------------- the kernel
template <int H, int I>
__global__ void __launch_bounds__(kThreads, 1) stack_decode2_kernel(const __grid_constant__ Params p) {
  constexpr int G = H / 64;
  constexpr int RGU = qrow_bytes(H, 4);   // gate/up record
  constexpr int RDN = qrow_bytes(I, 4);   // down record
  constexpr int UNIT = 4 * RGU;           // two (gate, up) row pairs
  constexpr int NCH_I = I / 32;           // int4 chunks per down row (one per lane of a segment)
  static_assert(H % 1024 == 0 && NCH_I <= 32 && (32 % NCH_I) == 0, "shape");
  constexpr int SEG = NCH_I;
  constexpr int SPW = 32 / SEG;           // down sub-rows per warp pass
  constexpr int HALF_I = I / 2;

  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ int s_idx[kMaxK];
  __shared__ float s_w[kMaxK];

  const Smem& S = p.sm;
  const int N = gridDim.x, c = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = p.K, E = p.E, r = p.r;
  int s0, s1, r0, r1, d0, d1, z0, z1, v0, v1;
  split(c, N, HALF_I, s0, s1);      // shared units (two pairs each)
  split(c, N, K * HALF_I, r0, r1);  // routed units
  split(c, N, H, d0, d1);           // output rows
  split(c, N, p.P, z0, z1);         // Prerouter hidden rows
  split(c, N, p.En, v0, v1);        // Prerouter output rows
  const int nS = s1 - s0, nR = r1 - r0, nD = d1 - d0, nZ = z1 - z0;

  // barriers: [0..1] static buffers, [2..2+maxR) routed units, then kMaxK down blocks
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S.bar);
  uint64_t* bar_unit = bar + 2;
  uint64_t* bar_down = bar + 2 + S.maxR;
  float* xs = reinterpret_cast<float*>(sm + S.xs);
  uint4* un = reinterpret_cast<uint4*>(sm + S.un);  // u, natural order fp16
  uint4* up = reinterpret_cast<uint4*>(sm + S.up);  // u, pair order fp16
  float* s16 = reinterpret_cast<float*>(sm + S.s16);
  float* s32 = reinterpret_cast<float*>(sm + S.s32);
  uint16_t* hs = reinterpret_cast<uint16_t*>(sm + S.hs);  // (K+1) x I fp16, pair order
  float* hsum = reinterpret_cast<float*>(sm + S.hsum);
  float* logit = reinterpret_cast<float*>(sm + S.logit);
  float* td = reinterpret_cast<float*>(sm + S.td);
  float* yd = reinterpret_cast<float*>(sm + S.yd);
  float* red = reinterpret_cast<float*>(sm + S.red);
  float* zx = reinterpret_cast<float*>(sm + S.zx);
  float* hloc = reinterpret_cast<float*>(sm + S.hloc);
  float* shacc = reinterpret_cast<float*>(sm + S.shacc);

  if (tid == 0) {
#pragma unroll 1
    for (int i = 0; i < 2 + S.maxR + kMaxK; ++i) mbar_init(bar + i);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  long long* trace = p.trace ? p.trace + static_cast<size_t>(c) * kTraceSlots : nullptr;
  auto stamp = [&](int l, int slot) {
    if (trace && tid == 0) trace[static_cast<size_t>(l) * N * kTraceSlots + slot] = gtimer();
  };

  uint32_t ph_st[2] = {0u, 0u}, ph_r = 0u;
  bool pend_st[2] = {false, false}, pend_r = false;
  bool ok = true;

  if (warp == kWarps - 1) issue_static<H, I>(p, sm, bar, 0, 0, s0, s1, d0, d1, z0, z1);
  pend_st[0] = true;

#pragma unroll 1
  for (int l = 0; l < p.n_layers && ok; ++l) {
    const LayerPtrs& L = p.L[l];
    const int b = l & 1;
    const uint32_t ep = static_cast<uint32_t>(l + 1);
    unsigned long long* llb = p.ll + static_cast<size_t>(b) * p.ll_stride;
    uint8_t* st = sm + S.st[b];

    // next layer's token-independent weights: its buffer was last read by layer l-1, which is done
    if (l + 1 < p.n_layers) {
      if (warp == kWarps - 1) issue_static<H, I>(p, sm, bar, l + 1, b ^ 1, s0, s1, d0, d1, z0, z1);
      pend_st[b ^ 1] = true;
    }
    // ================================================================ phase A: x -> u -> router rows
    if (l == 0) {
#pragma unroll 1
      for (int i = tid; i < H; i += kThreads) xs[i] = p.x[i];
      if (p.x_trace)
#pragma unroll 1
        for (int i = d0 + tid; i < d1; i += kThreads) p.x_trace[i] = p.x[i];
      __syncthreads();
    } else {
      const unsigned long long* xb = p.ll + static_cast<size_t>((l - 1) & 1) * p.ll_stride + p.ll_x;
      ok = gather(xb, H, static_cast<uint32_t>(l), p.timeout_ns, reinterpret_cast<uint32_t*>(xs));
      if (!ok) break;
    }
    stamp(l, 0);
    {  // RMSNorm -> bf16 -> fp16 (natural and pair order) + chunk sums; 4 values per thread
      float ss = 0.f;
#pragma unroll 1
      for (int i = tid; i < H; i += kThreads) ss = fmaf(xs[i], xs[i], ss);
      ss = warp_reduce(ss);
      if (lane == 0) red[warp] = ss;
      __syncthreads();
      float tot = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kWarps; ++w2) tot += red[w2];
      const float rs = rsqrtf(tot * (1.0f / static_cast<float>(H)) + p.eps);
      uint32_t* un32 = reinterpret_cast<uint32_t*>(un);
#pragma unroll 1
      for (int q4 = tid; q4 < H / 4; q4 += kThreads) {  // whole warps: H/4 is a multiple of 32
        const float4 xv = reinterpret_cast<const float4*>(xs)[q4];
        const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
        uint16_t e[4], bits[4];
        float bs = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          bits[i] = __bfloat16_as_ushort(__float2bfloat16_rn(xa[i] * rs));
          bs += bf16_bits_to_float(bits[i]);
          e[i] = bf16_to_f16_bits(bits[i]);
        }
        if (p.u_trace && c == 0) {
          uint2 tb;
          tb.x = bits[0] | (uint32_t(bits[1]) << 16);
          tb.y = bits[2] | (uint32_t(bits[3]) << 16);
          reinterpret_cast<uint2*>(p.u_trace + static_cast<size_t>(l) * H)[q4] = tb;
        }
        const uint32_t lo = e[0] | (uint32_t(e[1]) << 16), hi = e[2] | (uint32_t(e[3]) << 16);
        un32[2 * q4] = lo;
        un32[2 * q4 + 1] = hi;
        // pair order of the 8-block (q4/2): the even thread holds values 0..3, the odd one 4..7
        const uint32_t plo = __shfl_xor_sync(0xffffffffu, lo, 1), phi = __shfl_xor_sync(0xffffffffu, hi, 1);
        if ((q4 & 1) == 0)
          up[q4 >> 1] = make_uint4(prmt(lo, plo, 0x5410u), prmt(lo, plo, 0x7632u), prmt(hi, phi, 0x5410u),
                                   prmt(hi, phi, 0x7632u));
        bs += __shfl_xor_sync(0xffffffffu, bs, 1);
        bs += __shfl_xor_sync(0xffffffffu, bs, 2);  // 16 values
        if ((q4 & 3) == 0) s16[q4 >> 2] = bs;
        bs += __shfl_xor_sync(0xffffffffu, bs, 4);  // 32 values
        if ((q4 & 7) == 0) s32[q4 >> 3] = bs;
      }
    }
    // token-independent weights of this layer (the wait is also the barrier after the RMSNorm)
    ok = mbar_wait(bar + b, ph_st[b], p.timeout_ns);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    stamp(l, 1);
    ph_st[b] ^= 1u;
    pend_st[b] = false;
    {  // phase-A items: two per round, 256 threads each
      const int half = tid >> 8, t8 = tid & 255;
#pragma unroll 1
      for (int m0 = 0, i0 = c; i0 < p.NA; m0 += 2, i0 += 2 * N) {
        const int m = m0 + half, i = i0 + half * N;
        float acc = 0.f;
        if (i < p.NA) {
          const uint8_t* rec = st + S.o_items + m * S.item_bytes;
          if (i <= E) {  // 8-bit row: H/16 chunks of 16 codes
#pragma unroll 1
            for (int ch = t8; ch < H / 16; ch += 256) {
              const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + H);
              const int g = ch >> 2;
              const float s = half_bits_to_float(sc[g]);
              const float bb = half_bits_to_float(sc[G + g]) + 128.0f * s;
              const float d = dot_chunk_int8(reinterpret_cast<const uint4*>(rec)[ch], un + 2 * ch, 0.f);
              acc = fmaf(s, d, fmaf(bb, s16[ch], acc));
            }
          } else {  // fp16 LoRA A row: H/8 chunks
#pragma unroll 1
            for (int ch = t8; ch < H / 8; ch += 256) acc = dot_chunk_f16(reinterpret_cast<const uint4*>(rec)[ch], un[ch], acc);
          }
        }
        acc = warp_reduce(acc);
        if (lane == 0) red[warp] = acc;
        __syncthreads();
        if (t8 == 0 && i < p.NA) {
          float tot = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < 8; ++w2) tot += red[half * 8 + w2];
          if (i < E && L.rbias) tot += L.rbias[i];
          st_word(llb + p.ll_a + i, __float_as_uint(tot), ep);
        }
        __syncthreads();
      }
    }
    stamp(l, 2);
    // ---------------------------------------------------------------- while the logits travel
#pragma unroll 1
    for (int pi = warp; pi < 2 * nS; pi += kWarps) {  // shared (gate, up) base dot products
      float ag, au;
      pair_dots<H>(st + S.o_shu + (pi >> 1) * UNIT, pi & 1, up, s32, ag, au);
      if (lane == 0) {
        shacc[2 * pi] = ag;
        shacc[2 * pi + 1] = au;
      }
    }
    if (L.W1) {  // Prerouter hidden rows: the u part (the multi-hot part needs the executed experts)
      const int half = tid >> 8, t8 = tid & 255;
#pragma unroll 1
      for (int zz0 = z0; zz0 < z1; zz0 += 2) {
        const int zi = zz0 + half;
        float acc = 0.f;
        if (zi < z1) {
          const uint4* wr = reinterpret_cast<const uint4*>(st + S.o_W1 + (zi - z0) * 2 * H);
#pragma unroll 1
          for (int ch = t8; ch < H / 8; ch += 256) acc = dot_chunk_f16(wr[ch], un[ch], acc);
        }
        acc = warp_reduce(acc);
        if (lane == 0) red[warp] = acc;
        __syncthreads();
        if (t8 == 0 && zi < z1) {
          float tot = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < 8; ++w2) tot += red[half * 8 + w2];
          zx[zi - z0] = tot;
        }
        __syncthreads();
      }
    }
    stamp(l, 3);

    // ================================================================ phase B: top-K, gate/up + SwiGLU
    // the A words land contiguously: logits [0, E), shared-gate logit E, LoRA A u products after it
    ok = gather(llb + p.ll_a, p.NA, ep, p.timeout_ns, reinterpret_cast<uint32_t*>(logit));
    if (!ok) break;
    const float* tgu = logit + E + 1;
    stamp(l, 4);
    int e_lane;
    float w_lane;
    warp_select(logit, E, K, e_lane, w_lane, NoSlot{});  // every warp: lane k < K holds slot k's expert and weight
    if (warp == 0 && lane < K) {
      s_idx[lane] = e_lane;
      s_w[lane] = w_lane;
      if (c == 0) {
        if (p.idx_all) p.idx_all[static_cast<size_t>(l) * K + lane] = e_lane;
        if (p.true_idx_all) p.true_idx_all[static_cast<size_t>(l) * K + lane] = e_lane;
      }
    }
    stamp(l, 5);
    {  // routed-row copies, spread over the warps: copy j < nR is unit r0 + j, copy nR + k the down rows of slot k
      const RoutedCopies rc{L.pool, p.stride, sm + S.units, sm + S.down, bar_unit, bar_down, r0, nR,
                            nR + (nD > 0 ? K : 0), d0, nD, S.maxD, HALF_I, RGU, RDN, UNIT, 2 * I};
      pend_r = true;
#pragma unroll 1
      for (int j = warp; j < rc.ncopy; j += kWarps) rc.issue(j, __shfl_sync(0xffffffffu, e_lane, rc.slot(j)));
    }
    stamp(l, 6);
    {  // (gate, up) pairs: shared pairs get their LoRA delta; routed pairs as their rows land
      int wait_fail = 0;
#pragma unroll 1
      for (int pi = warp; pi < 2 * nS; pi += kWarps) {
        if (lane == 0) {
          float ag = shacc[2 * pi], au = shacc[2 * pi + 1];
          const int q = pi & 1;
          const uint16_t* Bb = reinterpret_cast<const uint16_t*>(st + S.o_shB + (pi >> 1) * 8 * r);
          if (L.Bg) {
            float d = 0.f;
#pragma unroll 1
            for (int i = 0; i < r; ++i) d = fmaf(half_bits_to_float(Bb[q * r + i]), tgu[i], d);
            ag = fmaf(p.lora_scale, d, ag);
          }
          if (L.Bu) {
            float d = 0.f;
#pragma unroll 1
            for (int i = 0; i < r; ++i) d = fmaf(half_bits_to_float(Bb[2 * r + q * r + i]), tgu[r + i], d);
            au = fmaf(p.lora_scale, d, au);
          }
          hloc[pi] = silu(ag) * au;
        }
      }
#pragma unroll 1
      for (int pi = warp; pi < 2 * nR; pi += kWarps) {
        const int uloc = pi >> 1;
        if (!mbar_wait(bar_unit + uloc, ph_r, p.timeout_ns)) wait_fail = 1;
        if (pi == 0 && lane == 0 && trace)  // the first routed pair's rows have landed
          trace[static_cast<size_t>(l) * N * kTraceSlots + 15] = gtimer();
        float ag, au;
        pair_dots<H>(sm + S.units + uloc * UNIT, pi & 1, up, s32, ag, au);
        if (lane == 0) hloc[2 * nS + pi] = silu(ag) * au;
      }
      ok = !__syncthreads_or(wait_fail);
      if (!ok) break;
    }
    stamp(l, 7);
    // publish h (one word per unit: two fp16 values) and the Prerouter hidden values
    if (tid < nS + nR) {
      const int i = tid;
      const uint32_t h2 = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hloc[2 * i]))) |
                          (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hloc[2 * i + 1]))) << 16);
      const int word = i < nS ? K * HALF_I + s0 + i : r0 + (i - nS);
      st_word(llb + p.ll_h + word, h2, ep);
    } else if (L.W1 && tid >= 32 * (kWarps - 1) && lane < nZ) {
      const int zi = z0 + lane;
      const uint16_t* row = L.W1 + static_cast<size_t>(zi) * (H + E) + H;
      float m = 0.f;
#pragma unroll 1
      for (int k = 0; k < K; ++k) m += half_bits_to_float(row[s_idx[k]]);
      st_word(p.ll + p.ll_z + static_cast<size_t>(l) * p.P + zi,
              __float_as_uint(silu(zx[lane] + m + half_bits_to_float(L.b1[zi]))), ep);
    }
    const float gate = sigmoid(logit[E]);  // shared-expert gate, while the hidden vector travels
    stamp(l, 8);

    // ================================================================ phase C: down projections + combine
    ok = gather_h(llb + p.ll_h, (K + 1) * HALF_I, HALF_I, ep, p.timeout_ns, hs, hsum);
    if (!ok) break;
    stamp(l, 9);
#pragma unroll 1
    for (int q = warp; L.Bd && q < r; q += kWarps) {  // t_d = A_d h_shared, one warp per rank
      const uint16_t* A = reinterpret_cast<const uint16_t*>(st + S.o_Ad) + static_cast<size_t>(q) * I;
      const uint16_t* h = hs + K * I;
      float acc = 0.f;
#pragma unroll 1
      for (int ch = lane; ch < I / 8; ch += 32) {
        const uint4 w = reinterpret_cast<const uint4*>(A)[ch];
        const uint4 hv = reinterpret_cast<const uint4*>(h)[ch];
        acc = dot2_mix(prmt(w.x, w.z, 0x5410u), hv.x, acc);
        acc = dot2_mix(prmt(w.x, w.z, 0x7632u), hv.y, acc);
        acc = dot2_mix(prmt(w.y, w.w, 0x5410u), hv.z, acc);
        acc = dot2_mix(prmt(w.y, w.w, 0x7632u), hv.w, acc);
      }
      acc = warp_reduce(acc);
      if (lane == 0) td[q] = acc;
    }
    int dfail = 0;  // every warp checks the routed down rows before reading them
#pragma unroll 1
    for (int k = 0; nD > 0 && k < K; ++k)
      if (!mbar_wait(bar_down + k, ph_r, p.timeout_ns)) dfail = 1;
    stamp(l, 10);
    if (!dfail) {  // down sub-rows: task = (row i, slot k), SEG lanes each, two independent tasks per pass
      const int ntask = nD * (K + 1);
      const int sub = lane / SEG, sl = lane % SEG;
      const int g = sl >> 1;
#pragma unroll 1
      for (int t0 = warp * SPW; t0 < ntask; t0 += 2 * kWarps * SPW) {
        float y[2];
        int ti[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int t = t0 + h * kWarps * SPW + sub;
          ti[h] = t;
          y[h] = 0.f;
          if (t < ntask) {
            const int i = t / (K + 1), k = t % (K + 1);
            const uint8_t* rec = k < K ? sm + S.down + (k * S.maxD + i) * RDN : st + S.o_sdn + i * RDN;
            const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + I / 2);
            const float s = half_bits_to_float(sc[g]);
            const float bb = half_bits_to_float(sc[I / 64 + g]) + 8.0f * s;
            const uint4 wv = reinterpret_cast<const uint4*>(rec)[sl];
            y[h] = fmaf(s, dot_chunk_int4(wv, reinterpret_cast<const uint4*>(hs + k * I) + 4 * sl, 0.f),
                        bb * hsum[k * NCH_I + sl]);
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float v = seg_reduce<SEG>(y[h]);
          const int t = ti[h];
          if (t < ntask && sl == 0) yd[(t / (K + 1)) * (K + 1) + t % (K + 1)] = v;
        }
      }
    }
    ok = !__syncthreads_or(dfail);
    if (!ok) break;
    ph_r ^= 1u;
    pend_r = false;
    stamp(l, 11);
    const bool last = l + 1 == p.n_layers;
    {  // combine: 16 lanes per output row (the shared down LoRA B row), then sum_k w_k y_k (k order) + g (y_s + LoRA)
      const int i = 2 * warp + (lane >> 4), q = lane & 15;
      float d = 0.f;
      if (L.Bd && i < nD) {
        const uint16_t* Br = reinterpret_cast<const uint16_t*>(st + S.o_Bd) + static_cast<size_t>(i) * r;
#pragma unroll 1
        for (int qq = q; qq < r; qq += 16) d = fmaf(half_bits_to_float(Br[qq]), td[qq], d);
      }
      d = seg_reduce<16>(d);
      if (q == 0 && i < nD) {
        const int o = d0 + i;
        float y = 0.f;
#pragma unroll 1
        for (int k = 0; k < K; ++k) y = fmaf(s_w[k], yd[i * (K + 1) + k], y);
        const float ys = fmaf(p.lora_scale, d, yd[i * (K + 1) + K]);
        const float xn = xs[o] + fmaf(gate, ys, y);
        if (!(l == p.drop_layer && c == p.drop_cta)) st_word(llb + p.ll_x + o, __float_as_uint(xn), ep);
        if (last) p.x[o] = xn;
        else if (p.x_trace) p.x_trace[static_cast<size_t>(l + 1) * H + o] = xn;
      }
    }
    __syncthreads();
    stamp(l, 12);
  }

  if (ok && p.L[0].W1)  // every Prerouter head's output layer and prediction, in the static buffers' space
    ok = prerouter_tail(p, v0, v1, reinterpret_cast<float*>(sm + S.st[0]), 2 * p.st_bytes / 4, logit);
  if (!ok) {
    if (tid == 0) atomicExch(p.err, 5);
  }
  // never leave with bulk copies in flight into this CTA's shared memory
  if (tid == 0) {
    for (int b2 = 0; b2 < 2; ++b2)
      if (pend_st[b2]) mbar_wait(bar + b2, ph_st[b2], 100000000LL);
    if (pend_r) {
#pragma unroll 1
      for (int i = 0; i < nR; ++i) mbar_wait(bar_unit + i, ph_r, 100000000LL);
      if (nD > 0)
#pragma unroll 1
        for (int k = 0; k < K; ++k) mbar_wait(bar_down + k, ph_r, 100000000LL);
    }
  }
  __syncthreads();
}

}  // namespace stk2
}  // namespace moe
