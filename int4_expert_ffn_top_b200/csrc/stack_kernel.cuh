// Persistent fused decode of a whole MoE stack for one token (batch 1).
//
// One cooperative launch runs every layer.  Each CTA (one per SM) owns fixed
// slices of every step: router rows / shared-gate / LoRA-A rows (phase A),
// gate/up row pairs of the routed and shared experts (phase B), output rows of
// the down projections and the combine (phase C), and Prerouter rows.
//
// Data movement:
// * weights that do not depend on the token (router, shared expert, its LoRA,
//   Prerouter) are prefetched two layers ahead into a double-buffered shared
//   memory region with 1-D TMA bulk copies (cp.async.bulk, mbarrier tx-count);
// * routed-expert rows are fetched the same way as soon as the CTA knows the
//   top-K -- one bulk copy per unit of work, because the expert block stores
//   each row (and each run of rows a unit needs) contiguously;
// * the three all-to-all exchanges per layer (logits, SwiGLU hidden vector,
//   residual stream) go through "epoch words": 64-bit global words holding a
//   32-bit payload and the 32-bit epoch of the layer that wrote it, stored and
//   loaded with single-copy-atomic 64-bit accesses, so a reader that sees the
//   epoch also sees the payload (one L2 round trip per exchange, no flags).
// Every wait is bounded by the global timer; on timeout the CTA records
// MOE_ERR_TIMEOUT, waits (bounded) for its own bulk copies and returns.
#pragma once

#include "common.cuh"

namespace moe {
namespace stk {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxLayers = 64;
constexpr int kTraceSlots = 16;  // see moe_stack_opts.trace

struct LayerPtrs {
  const uint8_t* router;  // E records (8-bit)
  const float* rbias;     // [E] or null
  const uint8_t* sgate;   // 1 record (8-bit)
  const uint8_t* shared;  // shared expert block
  const uint16_t *Ag, *Bg, *Au, *Bu, *Ad, *Bd;  // shared LoRA (null = none)
  const uint8_t* pool;
  const uint16_t *W1, *b1, *W2, *b2;  // Prerouter (null W1 = no head)
};

// Byte offsets into dynamic shared memory (computed on the host).
struct Smem {
  uint32_t st[2];                                             // static (token-independent) buffers
  uint32_t o_items, o_shu, o_shB, o_sdn, o_Bd, o_Ad, o_W1;  // offsets inside a static buffer
  uint32_t units, down;                                       // routed rows
  uint32_t xs, un, up, s16, s32, hs, hraw, hsum, logit, td, yd, red, z, hloc, bar, sent;
  uint32_t total;
  int maxA, maxS, maxR, maxD, maxZ, maxP, item_bytes;
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
  int ll_x, ll_a, ll_h, ll_z, ll_stride;  // per-parity regions; Prerouter scores of layer l at ll_p + l*En
  int ll_p;
  long long timeout_ns;
  int drop_layer, drop_cta;  // test hook: that CTA never publishes its residual rows of that layer
  long long* trace;          // optional [n_layers][grid][kTraceSlots] globaltimer stamps
  Smem sm;
  LayerPtrs L[kMaxLayers];
};

// ----------------------------------------------------------------------------- primitives
MOE_DEV uint32_t saddr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

MOE_DEV void mbar_init(uint64_t* b) { asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(b))); }

MOE_DEV void mbar_expect(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes) : "memory");
}

MOE_DEV bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

MOE_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   saddr(dst)),
               "l"(src), "r"(bytes), "r"(saddr(bar))
               : "memory");
}

MOE_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

MOE_DEV long long gtimer() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

MOE_DEV void st_word(unsigned long long* p, uint32_t payload, uint32_t epoch) {
  const unsigned long long v = (static_cast<unsigned long long>(epoch) << 32) | payload;
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

MOE_DEV unsigned long long ld_word(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Block-wide poll of n epoch words; take(i, payload) is called for every word
// carrying `epoch` (possibly more than once).  False on timeout (uniform).
template <typename F>
MOE_DEV bool poll_words(const unsigned long long* buf, int n, uint32_t epoch, long long timeout_ns, F take) {
  const long long deadline = gtimer() + timeout_ns;
  for (;;) {
    int ok = 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const unsigned long long v = ld_word(buf + i);
      if (static_cast<uint32_t>(v >> 32) == epoch) take(i, static_cast<uint32_t>(v));
      else ok = 0;
    }
    if (__syncthreads_and(ok)) return true;
    const int late = threadIdx.x == 0 && gtimer() > deadline;
    if (__syncthreads_or(late)) return false;
  }
}

// Two-stage block-wide poll: warp 0 first watches one sentinel word per
// producer (sent[0..ns), word indices) with a short back-off, then every thread
// reads all n words once (repeated only for words not yet visible).  Keeps the
// polling traffic on the lines producers are writing to ~one load per producer.
template <typename F>
MOE_DEV bool poll_words_sent(const unsigned long long* buf, int n, const int* sent, int ns, uint32_t epoch,
                             long long timeout_ns, F take) {
  const long long deadline = gtimer() + timeout_ns;
  int late = 0;
  if (threadIdx.x < 32) {
    for (int it = 0;; ++it) {
      int ok = 1;
      for (int i = threadIdx.x; i < ns; i += 32)
        if (static_cast<uint32_t>(ld_word(buf + sent[i]) >> 32) != epoch) ok = 0;
      if (__all_sync(0xffffffffu, ok)) break;
      if ((it & 15) == 15 && __any_sync(0xffffffffu, threadIdx.x == 0 && gtimer() > deadline)) {
        late = 1;
        break;
      }
      __nanosleep(32);
    }
  }
  if (__syncthreads_or(late)) return false;
  return poll_words(buf, n, epoch, timeout_ns, take);
}

#ifndef MOE_POLL_SENTINEL
#define MOE_POLL_SENTINEL 0  // 1: two-stage sentinel poll; 0: every thread polls its share of the words
#endif

// Out-of-line block-wide poll that stores the payloads of words [0, n) to dst.
__device__ __noinline__ bool poll_copy(const unsigned long long* buf, int n, const int* sent, int ns, uint32_t epoch,
                                       long long timeout_ns, uint32_t* dst) {
#if MOE_POLL_SENTINEL
  return poll_words_sent(buf, n, sent, ns, epoch, timeout_ns, [&](int i, uint32_t v) { dst[i] = v; });
#else
  (void)sent;
  (void)ns;
  return poll_words(buf, n, epoch, timeout_ns, [&](int i, uint32_t v) { dst[i] = v; });
#endif
}

// Warp-wide version (used by one warp while the others work).
template <typename F>
MOE_DEV bool poll_words_warp(const unsigned long long* buf, int n, uint32_t epoch, long long timeout_ns, F take) {
  const int lane = threadIdx.x & 31;
  const long long deadline = gtimer() + timeout_ns;
  for (;;) {
    int ok = 1;
    for (int i = lane; i < n; i += 32) {
      const unsigned long long v = ld_word(buf + i);
      if (static_cast<uint32_t>(v >> 32) == epoch) take(i, static_cast<uint32_t>(v));
      else ok = 0;
    }
    if (__all_sync(0xffffffffu, ok)) return true;
    if (__any_sync(0xffffffffu, lane == 0 && gtimer() > deadline)) return false;
  }
}

MOE_DEV bool mbar_wait(uint64_t* b, uint32_t parity, long long timeout_ns) {
  if (mbar_test(b, parity)) return true;
  const long long deadline = gtimer() + timeout_ns;
  for (int it = 1;; ++it) {
    if (mbar_test(b, parity)) return true;
    if ((it & 63) == 0 && gtimer() > deadline) return false;
  }
}

// Contiguous share [a, b) of n items for CTA c of N (c*n stays far below 2^31 here).
MOE_DEV void split(int c, int N, int n, int& a, int& b) {
  a = (c * n) / N;
  b = ((c + 1) * n) / N;
}

// Order-preserving map of a float to an unsigned key (larger float -> larger key).
MOE_DEV uint32_t ord_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
MOE_DEV float key_value(uint32_t k) { return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k); }

struct NoIssue {
  MOE_DEV void operator()(int, int) const {}
};

// Routed-row copies of one selected expert (slot k = expert e), spread over the
// lanes of the calling warp: this CTA's (gate, up) units of slot k and its
// down-row block of expert e.  The mbarriers were armed before the top-K.
struct RoutedIssue {
  const uint8_t* pool;
  int64_t stride;
  uint8_t* units;
  uint8_t* down;
  uint64_t* bar_unit;
  uint64_t* bar_down;
  int r0, r1, d0, nD, maxD, half_i, rgu, rdn, unit, i2;
  MOE_DEV void operator()(int k, int e) const {
    const int lane = threadIdx.x & 31;
    const uint8_t* blk = pool + static_cast<int64_t>(e) * stride;
    const int u0 = max(r0, k * half_i), u1 = min(r1, (k + 1) * half_i);
    int t = 0;
    for (int u = u0; u < u1; ++u, ++t)
      if (t % 32 == lane)
        bulk_load(units + (u - r0) * unit, blk + static_cast<size_t>(4 * (u - k * half_i)) * rgu, unit,
                  bar_unit + (u - r0));
    if (nD && t % 32 == lane)
      bulk_load(down + k * maxD * rdn, blk + static_cast<size_t>(i2) * rgu + static_cast<size_t>(d0) * rdn, nD * rdn,
                bar_down);
  }
};

template <typename Issue>
MOE_DEV void warp_topk_impl(const float* sc, int E, int K, int* sel, float* w, const Issue& issue) {
  const int lane = threadIdx.x & 31;
  uint32_t key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = lane + 32 * j;
    float x = i < E ? sc[i] : -INFINITY;
    if (x != x) x = -INFINITY;  // NaN ranks with -inf
    key[j] = i < E ? ord_key(x) : 0u;  // 0 is below every real key
  }
  uint32_t bk = key[0];
  int bj = 0;
#pragma unroll
  for (int j = 1; j < 8; ++j)
    if (key[j] > bk) {  // strict: the lowest j wins among equal keys of this lane
      bk = key[j];
      bj = j;
    }
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t win = __reduce_min_sync(0xffffffffu, bk == m ? static_cast<uint32_t>(lane + 32 * bj) : 0xffffffffu);
    if (static_cast<int>(win & 31u) == lane) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j == static_cast<int>(win >> 5)) key[j] = 0u;
      bk = key[0];
      bj = 0;
#pragma unroll
      for (int j = 1; j < 8; ++j)
        if (key[j] > bk) {
          bk = key[j];
          bj = j;
        }
    }
    const int e = static_cast<int>(win) < E ? static_cast<int>(win) : 0;
    issue(k, e);  // start fetching this expert's rows right away
    if (lane == 0) {
      sel[k] = e;
      if (w) w[k] = key_value(m);
    }
  }
  if (w && lane == 0) {  // softmax over the selected, summed in k order
    const float m0 = w[0];
    float sum = 0.f;
    for (int k = 0; k < K; ++k) {
      w[k] = expf(w[k] - m0);
      sum += w[k];
    }
    const float inv = __fdividef(1.0f, sum);
    for (int k = 0; k < K; ++k) w[k] *= inv;
  }
  __syncwarp();
}

// Top-K over E <= 256 scores in shared memory by one warp (descending, ties ->
// lower index); optional softmax over the selected.  Each round is one
// warp-wide max of the order keys and one min of the candidate indices
// (single-instruction warp reductions); only the winning lane rescans its 8
// values.  Lane 0 writes sel/w (shared memory).  Out of line: one warp runs
// it once per layer.
__device__ __noinline__ void warp_topk(const float* sc, int E, int K, int* sel, float* w) {
  warp_topk_impl(sc, E, K, sel, w, NoIssue{});
}

// Router top-K that issues each selected expert's routed-row copies as soon as
// that expert is known.
__device__ __noinline__ void warp_topk_issue(const float* sc, int E, int K, int* sel, float* w, const RoutedIssue& ri) {
  warp_topk_impl(sc, E, K, sel, w, ri);
}

// Issue the token-independent weights of layer l into static buffer b
// (called by warp 0; one bulk copy per lane per task).
struct Ranges {
  int s0, s1, d0, d1, z0, z1, v0, v1;
};

template <int H, int I>
__device__ __noinline__ void issue_static(const Params& p, uint8_t* sm, uint64_t* bar, int l, int b, const Ranges& rg) {
  constexpr int RGU = qrow_bytes(H, 4), RDN = qrow_bytes(I, 4), R8 = qrow_bytes(H, 8), UNIT = 4 * RGU;
  const Smem& S = p.sm;
  const int c = blockIdx.x, N = gridDim.x, lane = threadIdx.x & 31, E = p.E, r = p.r;
  const int nS = rg.s1 - rg.s0, nD = rg.d1 - rg.d0;
  const LayerPtrs& L = p.L[l];
  uint8_t* base = sm + S.st[b];
  uint32_t bytes = 0;
  for (int i = c; i < p.NA; i += N) bytes += i < E + 1 ? R8 : 2 * H;
  bytes += nS * UNIT + nD * RDN;
  if (L.Bg) bytes += nS * 4 * r;
  if (L.Bu) bytes += nS * 4 * r;
  if (L.Bd) bytes += nD * 2 * r + r * I * 2;
  if (L.W1) bytes += (rg.z1 - rg.z0) * 2 * H;
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
    task(base + S.o_shu + s * UNIT, L.shared + static_cast<size_t>(4 * (rg.s0 + s)) * RGU, UNIT);
    if (L.Bg) task(base + S.o_shB + s * 8 * r, L.Bg + static_cast<size_t>(2 * (rg.s0 + s)) * r, 4 * r);
    if (L.Bu) task(base + S.o_shB + s * 8 * r + 4 * r, L.Bu + static_cast<size_t>(2 * (rg.s0 + s)) * r, 4 * r);
  }
  task(base + S.o_sdn, L.shared + static_cast<size_t>(2 * I) * RGU + static_cast<size_t>(rg.d0) * RDN, nD * RDN);
  if (L.Bd) {
    task(base + S.o_Bd, L.Bd + static_cast<size_t>(rg.d0) * r, nD * 2 * r);
    task(base + S.o_Ad, L.Ad, r * I * 2);
  }
  if (L.W1) {
#pragma unroll 1
    for (int z = rg.z0; z < rg.z1; ++z)
      task(base + S.o_W1 + (z - rg.z0) * 2 * H, L.W1 + static_cast<size_t>(z) * (H + E), 2 * H);
  }
}

// Second Prerouter layer of layer lp for rows [v0, v1): p_e = W2[e] . z + b2[e]
// with z the (complete) hidden vector of that head; W2 rows are read directly.
template <int H>
__device__ __noinline__ bool prerouter_out(const Params& p, int lp, int v0, int v1, float* zs, const int* sent_z,
                                           int nsz) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned long long* zb = p.ll + static_cast<size_t>(lp & 1) * p.ll_stride + p.ll_z;
  const uint32_t epoch = static_cast<uint32_t>(lp + 1);
  if (!poll_copy(zb, p.P, sent_z, nsz, epoch, p.timeout_ns, reinterpret_cast<uint32_t*>(zs))) return false;
  const LayerPtrs& L = p.L[lp];
  unsigned long long* pb = p.ll + p.ll_p + static_cast<size_t>(lp) * p.En;
#pragma unroll 1
  for (int e = v0 + warp; e < v1; e += blockDim.x / 32) {
    const uint4* w2 = reinterpret_cast<const uint4*>(L.W2 + static_cast<size_t>(e) * p.P);
    float acc = 0.f;
#pragma unroll 1
    for (int ch = lane; ch < p.P / 8; ch += 32) {
      const uint4 w = w2[ch];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 f = __half22float2(as_h2(ws[m]));
        acc = fmaf(f.x, zs[ch * 8 + 2 * m], acc);
        acc = fmaf(f.y, zs[ch * 8 + 2 * m + 1], acc);
      }
    }
    acc = warp_reduce(acc);
    if (lane == 0) st_word(pb + e, __float_as_uint(acc + half_bits_to_float(L.b2[e])), epoch);
  }
  __syncthreads();
  return true;
}

// Prediction of head lp (one warp): top-K of its published scores -> pred_all[lp].
__device__ __noinline__ void predict(const Params& p, int lp, float* scratch, int* sel) {
  const int lane = threadIdx.x & 31;
  const unsigned long long* pb = p.ll + p.ll_p + static_cast<size_t>(lp) * p.En;
  if (poll_words_warp(pb, p.En, static_cast<uint32_t>(lp + 1), p.timeout_ns,
                      [&](int i, uint32_t v) { scratch[i] = __uint_as_float(v); })) {
    __syncwarp();
    warp_topk(scratch, p.En, p.K, sel, nullptr);
    if (lane < p.K && p.pred_all) p.pred_all[static_cast<size_t>(lp) * p.K + lane] = sel[lane];
  } else if (lane == 0) {
    atomicExch(p.err, 5);
  }
}

// ----------------------------------------------------------------------------- the kernel
template <int H, int I>
__global__ void __launch_bounds__(kThreads, 1) stack_decode_kernel(const __grid_constant__ Params p) {
  constexpr int G = H / 64;
  constexpr int RGU = qrow_bytes(H, 4);   // gate/up record
  constexpr int RDN = qrow_bytes(I, 4);   // down record
  constexpr int R8 = qrow_bytes(H, 8);    // router / shared-gate record
  constexpr int UNIT = 4 * RGU;           // two (gate, up) row pairs
  constexpr int CPL = (H / 32) / 32;      // int4 chunks per lane per gate/up row
  constexpr int NCH_I = I / 32;           // int4 chunks per down row (one per lane of a segment)
  static_assert(H % 1024 == 0 && NCH_I <= 32 && (32 % NCH_I) == 0, "shape");
  constexpr int SEG = NCH_I;
  constexpr int SPW = 32 / SEG;           // down sub-rows per warp pass

  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ int s_idx[8];
  __shared__ float s_w[8];
  __shared__ int s_pred[8];

  const Smem& S = p.sm;
  const int N = gridDim.x, c = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = p.K, E = p.E, r = p.r;
  const int HALF_I = I / 2;
  int s0, s1, r0, r1, d0, d1, z0, z1, v0, v1;
  split(c, N, HALF_I, s0, s1);      // shared units (two pairs each)
  split(c, N, K * HALF_I, r0, r1);  // routed units
  split(c, N, H, d0, d1);           // output rows
  split(c, N, p.P, z0, z1);         // Prerouter hidden rows
  split(c, N, p.En, v0, v1);        // Prerouter output rows
  const int nS = s1 - s0, nR = r1 - r0, nD = d1 - d0;

  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + S.bar);  // [0..1] static, [2..2+maxR) units, [2+maxR] down
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
  float* zs = reinterpret_cast<float*>(sm + S.z);
  float* hloc = reinterpret_cast<float*>(sm + S.hloc);

  // sentinel words: one per producing CTA of each exchanged buffer
  int* sent_x = reinterpret_cast<int*>(sm + S.sent);
  int* sent_a = sent_x + N;
  int* sent_h = sent_a + N;
  int* sent_z = sent_h + 2 * N;
  int* sent_p = sent_z + N;
  __shared__ int s_ns[5];
  if (tid == 0) {
    #pragma unroll 1
    for (int i = 0; i < 3 + S.maxR; ++i) mbar_init(bar + i);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    int nx = 0, na = 0, nh = 0, nz = 0, np = 0;
    #pragma unroll 1
    for (int q = 0; q < N; ++q) {
      int a0, a1;
      split(q, N, H, a0, a1);
      if (a1 > a0) sent_x[nx++] = a0;
      if (q < p.NA) sent_a[na++] = q;
      split(q, N, K * HALF_I, a0, a1);
      if (a1 > a0) sent_h[nh++] = a0;
      split(q, N, HALF_I, a0, a1);
      if (a1 > a0) sent_h[nh++] = K * HALF_I + a0;
      split(q, N, p.P, a0, a1);
      if (a1 > a0) sent_z[nz++] = a0;
      split(q, N, p.En, a0, a1);
      if (a1 > a0) sent_p[np++] = a0;
    }
    s_ns[0] = nx;
    s_ns[1] = na;
    s_ns[2] = nh;
    s_ns[3] = nz;
    s_ns[4] = np;
  }
  __syncthreads();
  long long* trace = p.trace ? p.trace + static_cast<size_t>(c) * kTraceSlots : nullptr;
  auto stamp = [&](int l, int slot) {
    if (trace && tid == 0) trace[static_cast<size_t>(l) * N * kTraceSlots + slot] = gtimer();
  };

  uint32_t ph_st[2] = {0u, 0u}, ph_unit = 0u, ph_down = 0u;
  bool pend_st[2] = {false, false}, pend_unit = false, pend_down = false;
  bool ok = true;

  const Ranges rgs{s0, s1, d0, d1, z0, z1, v0, v1};
  if (warp == 0) issue_static<H, I>(p, sm, bar, 0, 0, rgs);
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
      if (warp == 0) issue_static<H, I>(p, sm, bar, l + 1, b ^ 1, rgs);
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
      ok = poll_copy(xb, H, sent_x, s_ns[0], static_cast<uint32_t>(l), p.timeout_ns, reinterpret_cast<uint32_t*>(xs));
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
      __syncthreads();
    }
    stamp(l, 8);
    // token-independent weights of this layer
    ok = mbar_wait(bar + b, ph_st[b], p.timeout_ns);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    stamp(l, 9);
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
            for (int ch = t8; ch < H / 8; ch += 256)
              acc = dot_chunk_f16(reinterpret_cast<const uint4*>(rec)[ch], un[ch], acc);
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
    stamp(l, 1);

    // ================================================================ phase B: top-K, gate/up + SwiGLU
    // the A words land contiguously: logits [0, E), shared-gate logit E, LoRA A u products after it
    ok = poll_copy(llb + p.ll_a, p.NA, sent_a, s_ns[1], ep, p.timeout_ns, reinterpret_cast<uint32_t*>(logit));
    if (!ok) break;
    const float* tgu_l = logit + E + 1;
    const float g_raw = logit[E];
    stamp(l, 2);
    if (warp == 0) {
      // arm the routed-row barriers, then select the experts, issuing each one's copies as soon as it is known
      fence_proxy_async();
      if (lane == 0) {
        #pragma unroll 1
        for (int i = 0; i < nR; ++i) mbar_expect(bar_unit + i, UNIT);
        mbar_expect(bar_down, static_cast<uint32_t>(K * nD * RDN));
      }
      __syncwarp();
      const RoutedIssue ri{L.pool, p.stride, sm + S.units, sm + S.down, bar_unit, bar_down, r0, r1, d0, nD, S.maxD,
                           HALF_I, RGU, RDN, UNIT, 2 * I};
      warp_topk_issue(logit, E, K, s_idx, s_w, ri);
      stamp(l, 10);
      if (lane < K && c == 0) {
        if (p.idx_all) p.idx_all[static_cast<size_t>(l) * K + lane] = s_idx[lane];
        if (p.true_idx_all) p.true_idx_all[static_cast<size_t>(l) * K + lane] = s_idx[lane];
      }
    }
    pend_unit = pend_down = true;  // the pair loop below waits on the unit barriers; no block barrier needed
    stamp(l, 3);
    {  // (gate, up) pairs: shared units first (already resident), then routed units as they land
      const int npairs = 2 * (nS + nR);
      int wait_fail = 0;
      #pragma unroll 1
      for (int pi = warp; pi < npairs; pi += kWarps) {
        const bool shared = pi < 2 * nS;
        const int uloc = shared ? pi >> 1 : (pi - 2 * nS) >> 1;
        const int q = pi & 1;
        const uint8_t* rec4 = shared ? st + S.o_shu + uloc * UNIT : sm + S.units + uloc * UNIT;
        if (!shared && !mbar_wait(bar_unit + uloc, ph_unit, p.timeout_ns)) wait_fail = 1;
        if (pi == 2 * nS && lane == 0 && trace)  // the first routed pair's rows have landed
          trace[static_cast<size_t>(l) * N * kTraceSlots + 13] = gtimer();
        const uint8_t* rg = rec4 + (2 * q) * RGU;
        const uint8_t* ru = rg + RGU;
        const uint16_t* sg = reinterpret_cast<const uint16_t*>(rg + H / 2);
        const uint16_t* su = reinterpret_cast<const uint16_t*>(ru + H / 2);
        float ag = 0.f, au = 0.f;
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
          const int ch = lane + 32 * cc, g = ch >> 1;
          const uint4 wg = reinterpret_cast<const uint4*>(rg)[ch];
          const uint4 wu = reinterpret_cast<const uint4*>(ru)[ch];
          const float us = s32[ch];
          const float sgv = half_bits_to_float(sg[g]), sug = half_bits_to_float(su[g]);
          ag = fmaf(sgv, dot_chunk_int4(wg, up + 4 * ch, 0.f),
                    fmaf(half_bits_to_float(sg[G + g]) + 8.0f * sgv, us, ag));
          au = fmaf(sug, dot_chunk_int4(wu, up + 4 * ch, 0.f),
                    fmaf(half_bits_to_float(su[G + g]) + 8.0f * sug, us, au));
        }
        ag = warp_reduce(ag);
        au = warp_reduce(au);
        if (lane == 0) {
          if (shared) {
            const uint16_t* Bb = reinterpret_cast<const uint16_t*>(st + S.o_shB + uloc * 8 * r);
            if (L.Bg) {
              float d = 0.f;
              #pragma unroll 1
              for (int i = 0; i < r; ++i) d = fmaf(half_bits_to_float(Bb[q * r + i]), tgu_l[i], d);
              ag = fmaf(p.lora_scale, d, ag);
            }
            if (L.Bu) {
              float d = 0.f;
              #pragma unroll 1
              for (int i = 0; i < r; ++i) d = fmaf(half_bits_to_float(Bb[2 * r + q * r + i]), tgu_l[r + i], d);
              au = fmaf(p.lora_scale, d, au);
            }
          }
          hloc[pi] = silu(ag) * au;
        }
      }
      ok = !__syncthreads_or(wait_fail);
      if (!ok) break;
      ph_unit ^= 1u;
      pend_unit = false;
      // publish h: one word per unit (two fp16 values)
      #pragma unroll 1
      for (int i = tid; i < nS + nR; i += kThreads) {
        const bool shared = i < nS;
        const int pi = 2 * i;
        const uint32_t h2 = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hloc[pi]))) |
                            (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hloc[pi + 1]))) << 16);
        const int word = shared ? K * HALF_I + s0 + i : r0 + (i - nS);
        st_word(llb + p.ll_h + word, h2, ep);
      }
    }
    stamp(l, 4);
    if (L.W1) {  // Prerouter hidden rows (off the critical path)
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
          const uint16_t* row = L.W1 + static_cast<size_t>(zi) * (H + E) + H;
          float m = 0.f;
          #pragma unroll 1
          for (int k = 0; k < K; ++k) m += half_bits_to_float(row[s_idx[k]]);
          st_word(llb + p.ll_z + zi, __float_as_uint(silu(tot + m + half_bits_to_float(L.b1[zi]))), ep);
        }
        __syncthreads();
      }
    }
    // ================================================================ phase C: down projections + combine
    {
      uint32_t* hraw = reinterpret_cast<uint32_t*>(sm + S.hraw);
      ok = poll_copy(llb + p.ll_h, (K + 1) * HALF_I, sent_h, s_ns[2], ep, p.timeout_ns, hraw);
      if (!ok) break;
      #pragma unroll 1
      for (int w = tid; w < (K + 1) * HALF_I; w += kThreads) {  // to pair order
        const uint32_t v = hraw[w];
        const int k = w / HALF_I, j = 2 * (w % HALF_I);
        hs[k * I + pair_pos(j)] = static_cast<uint16_t>(v & 0xffffu);
        hs[k * I + pair_pos(j + 1)] = static_cast<uint16_t>(v >> 16);
      }
      __syncthreads();
    }
    stamp(l, 5);
    #pragma unroll 1
    for (int ch = tid; ch < (K + 1) * I / 32; ch += kThreads) {  // sums of 32-element chunks
      const uint4* hp = reinterpret_cast<const uint4*>(hs) + ch * 4;
      float t = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = hp[i];
        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float2 f = __half22float2(as_h2(vv[m]));
          t += f.x + f.y;
        }
      }
      hsum[ch] = t;
    }
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
    stamp(l, 14);
    ok = mbar_wait(bar_down, ph_down, p.timeout_ns);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    stamp(l, 15);
    ph_down ^= 1u;
    pend_down = false;
    {  // down sub-rows: task = (row i, slot k), SEG lanes each
      const int ntask = nD * (K + 1);
      const int sub = lane / SEG, sl = lane % SEG;
      #pragma unroll 1
      for (int t0 = warp * SPW; t0 < ntask; t0 += kWarps * SPW) {
        const int t = t0 + sub;
        float y = 0.f;
        int i = 0, k = 0;
        if (t < ntask) {
          i = t / (K + 1);
          k = t % (K + 1);
          const uint8_t* rec = k < K ? sm + S.down + (k * S.maxD + i) * RDN : st + S.o_sdn + i * RDN;
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + I / 2);
          const int ch = sl, g = ch >> 1;
          const float s = half_bits_to_float(sc[g]);
          const float bb = half_bits_to_float(sc[I / 64 + g]) + 8.0f * s;
          const uint4 wv = reinterpret_cast<const uint4*>(rec)[ch];
          y = fmaf(s, dot_chunk_int4(wv, reinterpret_cast<const uint4*>(hs + k * I) + 4 * ch, 0.f),
                   bb * hsum[k * NCH_I + ch]);
        }
        y = seg_reduce<SEG>(y);
        if (t < ntask && sl == 0) yd[i * (K + 1) + k] = y;
      }
    }
    __syncthreads();
    const bool last = l + 1 == p.n_layers;
    const float gate = sigmoid(g_raw);
    #pragma unroll 1
    for (int i = warp; i < nD; i += kWarps) {  // one warp per output row
      const int o = d0 + i;
      float d = 0.f;
      if (L.Bd && lane < r)
        d = half_bits_to_float(reinterpret_cast<const uint16_t*>(st + S.o_Bd)[static_cast<size_t>(i) * r + lane]) *
            td[lane];
      d = warp_reduce(d);
      if (lane == 0) {
        float y = 0.f;
        #pragma unroll 1
        for (int k = 0; k < K; ++k) y = fmaf(s_w[k], yd[i * (K + 1) + k], y);  // fixed k order
        const float ys = fmaf(p.lora_scale, d, yd[i * (K + 1) + K]);
        const float xn = xs[o] + fmaf(gate, ys, y);
        if (!(l == p.drop_layer && c == p.drop_cta)) st_word(llb + p.ll_x + o, __float_as_uint(xn), ep);
        if (last) p.x[o] = xn;
        else if (p.x_trace) p.x_trace[static_cast<size_t>(l + 1) * H + o] = xn;
      }
    }
    __syncthreads();
    stamp(l, 6);
    if (L.W1 && l > 0) {  // second Prerouter layer of the previous layer, while the residual exchange is in flight
      ok = prerouter_out<H>(p, l - 1, v0, v1, zs, sent_z, s_ns[3]);
      if (!ok) break;
    }
    __syncthreads();
    stamp(l, 7);
  }

  if (ok && p.L[p.n_layers - 1].W1) {  // the last layer's second Prerouter layer and the outstanding predictions
    const int n = p.n_layers;
    ok = prerouter_out<H>(p, n - 1, v0, v1, zs, sent_z, s_ns[3]);
    // predictions of every head, spread over the CTAs (one warp each)
    if (ok && warp == 0)
#pragma unroll 1
      for (int lp = c; lp < n; lp += N) predict(p, lp, logit, s_pred);
  }
  if (!ok) {
    if (tid == 0) atomicExch(p.err, 5);
  }
  // never leave with bulk copies in flight into this CTA's shared memory
  if (tid == 0) {
    for (int b2 = 0; b2 < 2; ++b2)
      if (pend_st[b2]) mbar_wait(bar + b2, ph_st[b2], 100000000LL);
    if (pend_unit)
      #pragma unroll 1
      for (int i = 0; i < nR; ++i) mbar_wait(bar_unit + i, ph_unit, 100000000LL);
    if (pend_down) mbar_wait(bar_down, ph_down, 100000000LL);
  }
  __syncthreads();
}

}  // namespace stk
}  // namespace moe
