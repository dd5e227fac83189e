// C ABI of the routed-expert layer library: argument checks on the host, then
// kernel launches on the caller's stream.  Nothing here allocates memory.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/moe.h"
#include "dense_gemm.cuh"
#include "layer_kernels.cuh"
#include "prefill_kernels.cuh"
#include "stack_kernel.cuh"
#include "stack2_kernel.cuh"
#include "tier.cuh"

namespace {

using namespace moe;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// Supported hidden sizes and intermediate sizes (template instantiations).
inline bool h_ok(int H) { return pow2_in(H, 256, 4096); }
inline bool i_ok(int I) { return pow2_in(I, 128, 2048); }

moe_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

bool qrows_ok(const moe_qrows& m, int out_dim, int in_dim, int bits) {
  return m.rows && m.out_dim == out_dim && m.in_dim == in_dim && m.bits == bits && aligned(m.rows, 16);
}

moe_status check_layer(const moe_layer* L, int T, int K) {
  if (!L) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > MOE_MAX_TOKENS || K < 1 || K > 8) return MOE_ERR_UNSUPPORTED;
  if (!h_ok(L->H) || !i_ok(L->I) || L->I_s != L->I) return MOE_ERR_UNSUPPORTED;
  // LoRA rank a multiple of 8 (0: none): the LoRA tensors move in 16-byte units (bulk copies of 4r- and
  // 2r-byte row runs, 16-byte loads of B rows), which other ranks would misalign
  if (L->E < K || L->E > 256 || L->r < 0 || L->r > 32 || L->r % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!qrows_ok(L->router, L->E, L->H, 8)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

size_t block_bytes(int H, int I) {
  return static_cast<size_t>(2 * I) * qrow_bytes(H, 4) + static_cast<size_t>(H) * qrow_bytes(I, 4);
}

// Weight pointers moe_expert_forward reads besides the router (after check_layer).
moe_status check_expert_weights(const moe_layer* L) {
  if (!L->pool || !aligned(L->pool, 256) || L->expert_stride < static_cast<int64_t>(block_bytes(L->H, L->I)) ||
      L->expert_stride % 256)
    return MOE_ERR_INVALID_ARG;
  if (!qrows_ok(L->shared_gate, 1, L->H, 8) || !L->shared_block || !aligned(L->shared_block, 16))
    return MOE_ERR_INVALID_ARG;
  if (L->r > 0) {
    for (int p = 0; p < 3; ++p)
      if ((L->sh_lora_A[p] != nullptr) != (L->sh_lora_B[p] != nullptr)) return MOE_ERR_INVALID_ARG;
    if ((L->ex_lora_A != nullptr) != (L->ex_lora_B != nullptr)) return MOE_ERR_INVALID_ARG;
    if ((L->ex_lora_A_gu != nullptr) != (L->ex_lora_B_gu != nullptr)) return MOE_ERR_INVALID_ARG;
    const void* lp[10] = {L->sh_lora_A[0], L->sh_lora_A[1], L->sh_lora_A[2], L->ex_lora_A, L->ex_lora_A_gu,
                          L->sh_lora_B[0], L->sh_lora_B[1], L->sh_lora_B[2], L->ex_lora_B, L->ex_lora_B_gu};
    for (const void* p : lp)
      if (p && !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// Shapes a Prerouter head supports for (K, K_next).
moe_status check_head_shape(const moe_prerouter* P, int K, int K_next) {
  if (K < 1 || K > 8 || K_next < 1 || K_next > 8) return MOE_ERR_UNSUPPORTED;
  if (!h_ok(P->H) || P->E < K || P->E > 256 || P->E % 8 || P->E_next < K_next || P->E_next > 256 || P->P < 8 ||
      P->P % 8)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_head_weights(const moe_prerouter* P) {
  if (!P->W1 || !P->b1 || !P->W2 || !P->b2 || !aligned(P->W1, 16) || !aligned(P->W2, 16)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Workspace carve-up of moe_expert_forward.
struct Ws {
  void* base;
  int32_t *idx, *count, *offset, *perm, *inv;
  float *g, *t_gu, *t_ds, *t_ex;
  uint16_t* h16;
  size_t bytes;
};

Ws carve(void* base, int T, int K, int E, int I, int r) {
  Ws w{};
  w.base = base;
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off = align_up(off + n, 256);
    return base ? static_cast<char*>(base) + o : nullptr;
  };
  const size_t TK = static_cast<size_t>(T) * K;
  w.idx = reinterpret_cast<int32_t*>(take(TK * 4));
  w.count = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E) * 4));
  w.offset = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
  w.perm = reinterpret_cast<int32_t*>(take(TK * 4));
  w.inv = reinterpret_cast<int32_t*>(take(TK * 4));
  w.g = reinterpret_cast<float*>(take(static_cast<size_t>(T) * 4));
  w.t_gu = reinterpret_cast<float*>(take(static_cast<size_t>(T) * 2 * (r > 0 ? r : 1) * 4));
  w.t_ds = reinterpret_cast<float*>(take(static_cast<size_t>(T) * (r > 0 ? r : 1) * 4));
  w.t_ex = reinterpret_cast<float*>(take(TK * (r > 0 ? r : 1) * 4));
  w.h16 = reinterpret_cast<uint16_t*>(take((TK + T) * static_cast<size_t>(I) * 2));
  w.bytes = off;
  return w;
}

size_t gemv_smem(int H, bool sum32, bool sum16) {
  return static_cast<size_t>(TB) * H * 2 + (sum32 ? static_cast<size_t>(TB) * (H / 32) * 4 : 0) +
         (sum16 ? static_cast<size_t>(TB) * (H / 16) * 4 : 0);
}

template <typename KernelT>
void allow_smem(KernelT k, size_t bytes) {
  if (bytes > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

// Many-token batches of the router and the Prerouter's first layer run on the tensor cores (dense::dense_kernel)
// from this many tokens on; fewer take the CUDA-core GEMVs.
constexpr int kDenseMinTokens = 256;
bool dense_router_ok(const moe_layer* L, const uint16_t* u, int T);
moe_status dense_router(const moe_layer* L, const uint16_t* u, int T, float* logits, int* err, cudaStream_t st);
bool dense_w1_ok(const moe_prerouter* P, const uint16_t* u, int T);
moe_status dense_w1(const moe_prerouter* P, const uint16_t* u, const int32_t* sel, int T, int K, float* z, int* err,
                    cudaStream_t st);

template <int H>
moe_status route_h(const moe_layer* L, const uint16_t* u, int T, int K, float* logits, int32_t* idx, float* w,
                   int* err, cudaStream_t st) {
  if (dense_router_ok(L, u, T)) {
    const moe_status s = dense_router(L, u, T, logits, err, st);
    if (s != MOE_OK) return s;
    topk_kernel<<<(T + kWarps - 1) / kWarps, kThreads, 0, st>>>(logits, T, L->E, K, idx, w);
    return launch_status();
  }
  constexpr int NCH = H / 16;
  constexpr int SEG = NCH < 32 ? NCH : 32;
  const int rows_per_cta = kWarps * (32 / SEG);
  const size_t smem = gemv_smem(H, false, true);
  allow_smem(router_kernel<NCH>, smem);
  dim3 grid((L->E + rows_per_cta - 1) / rows_per_cta, (T + TB - 1) / TB);
  router_kernel<NCH><<<grid, kThreads, smem, st>>>(u, T, static_cast<const uint8_t*>(L->router.rows),
                                                   L->router_bias, L->E, logits, err);
  topk_kernel<<<(T + kWarps - 1) / kWarps, kThreads, 0, st>>>(logits, T, L->E, K, idx, w);
  return launch_status();
}

template <int H, int I>
moe_status expert_forward_hi(const moe_layer* L, const uint16_t* u, int T, int K, const int32_t* idx, const float* w,
                             void* out, int out_mode, int32_t* perm_out, const Ws& ws, int* err, cudaStream_t st) {
  const int TK = T * K;
  // 1) buckets, shared gate, shared LoRA A u
  PreArgs pa{};
  pa.u = u;
  pa.T = T;
  pa.K = K;
  pa.E = L->E;
  pa.r = L->r;
  pa.idx_in = idx;
  pa.idx = ws.idx;
  pa.perm_out = perm_out;
  pa.count = ws.count;
  pa.offset = ws.offset;
  pa.perm = ws.perm;
  pa.inv = ws.inv;
  pa.sg_rec = static_cast<const uint8_t*>(L->shared_gate.rows);
  pa.A_gate = L->r > 0 ? L->sh_lora_A[0] : nullptr;
  pa.A_up = L->r > 0 ? L->sh_lora_A[1] : nullptr;
  pa.g = ws.g;
  pa.t_gu = ws.t_gu;
  pa.err = err;
  const int nrows = 1 + (pa.A_gate ? L->r : 0) + (pa.A_up ? L->r : 0);
  const size_t smem_pre = gemv_smem(H, false, true);
  allow_smem(pre_kernel<H / 8>, smem_pre);
  pre_kernel<H / 8><<<1 + (nrows + kWarps - 1) / kWarps, kThreads, smem_pre, st>>>(pa);
  // 2) gate/up + SwiGLU for every touched expert and the shared expert
  GateUpArgs ga{};
  ga.u = u;
  ga.T = T;
  ga.K = K;
  ga.I = I;
  ga.idx = ws.idx;
  ga.perm = ws.perm;
  ga.offset = ws.offset;
  ga.pool = static_cast<const uint8_t*>(L->pool);
  ga.stride = L->expert_stride;
  ga.sh_block = static_cast<const uint8_t*>(L->shared_block);
  ga.sh_Bg = (L->r > 0 && L->sh_lora_A[0]) ? L->sh_lora_B[0] : nullptr;
  ga.sh_Bu = (L->r > 0 && L->sh_lora_A[1]) ? L->sh_lora_B[1] : nullptr;
  ga.t_gu = ws.t_gu;
  ga.r = L->r;
  ga.lora_scale = L->lora_scale;
  ga.h16 = ws.h16;
  ga.err = err;
  {
    constexpr int NCH = H / 32;
    constexpr int SEG = NCH < 32 ? NCH : 32;
    const int pairs_per_cta = kWarps * (32 / SEG);
    const size_t smem = gemv_smem(H, true, false);
    allow_smem(gate_up_kernel<NCH>, smem);
    dim3 grid((I + pairs_per_cta - 1) / pairs_per_cta, TK + 1);
    gate_up_kernel<NCH><<<grid, kThreads, smem, st>>>(ga);
  }
  // 3) LoRA A h for the shared down projection and routed down projections
  MidArgs ma{};
  ma.T = T;
  ma.K = K;
  ma.I = I;
  ma.r = L->r;
  ma.idx = ws.idx;
  ma.h16 = ws.h16;
  ma.A_sd = (L->r > 0) ? L->sh_lora_A[2] : nullptr;
  ma.A_ex = (L->r > 0) ? L->ex_lora_A : nullptr;
  ma.t_ds = ws.t_ds;
  ma.t_ex = ws.t_ex;
  const int n_mid = (ma.A_sd ? T * L->r : 0) + (ma.A_ex ? TK * L->r : 0);
  if (n_mid > 0) lora_mid_kernel<<<(n_mid + kWarps - 1) / kWarps, kThreads, 0, st>>>(ma);
  // 4) down projections + combine
  DownArgs da{};
  da.T = T;
  da.K = K;
  da.H = H;
  da.I = I;
  da.r = L->r;
  da.idx = ws.idx;
  da.w = w;
  da.g = ws.g;
  da.pool = static_cast<const uint8_t*>(L->pool);
  da.stride = L->expert_stride;
  da.sh_block = static_cast<const uint8_t*>(L->shared_block);
  da.B_sd = ma.A_sd ? L->sh_lora_B[2] : nullptr;
  da.B_ex = ma.A_ex ? L->ex_lora_B : nullptr;
  da.t_ds = ws.t_ds;
  da.t_ex = ws.t_ex;
  da.lora_scale = L->lora_scale;
  da.h16 = ws.h16;
  da.out = out;
  da.out_mode = out_mode;
  down_kernel<I / 32><<<(H + kWarps - 1) / kWarps, kThreads, 0, st>>>(da);
  return launch_status();
}

// ----------------------------------------------------------------------------- grouped-GEMM path (many slots)
// T*K from which moe_expert_forward uses the tensor-core path.  Measured on the 35B layer shape (K = 4): the
// GEMVs are faster up to 8 tokens (32 slots: 93 us against 103 us), the grouped GEMMs from 16 tokens (64 slots:
// 121 us against 170 us); mean slots per touched expert stays between 1.0 and 1.9 over that range, so it does
// not separate the two, while the slot count does.
constexpr int kGemmMinSlots = 48;
constexpr long long kGemmTimeoutNs = 2000000000LL;  // bound of every wait of the grouped GEMMs

struct GWs {
  int32_t *idx, *count, *offset, *perm, *inv, *blockhist;
  float *w_pos, *t1, *t2, *g;
  uint16_t *X, *Hh, *Y;
  uint16_t* D;  // the shared expert's per-token LoRA deltas: gate/up [T][2I], then (reused) down [T][H]
  float* tv;    // their per-token LoRA-A products: gate/up [T][2r], then (reused) down [T][r]
  tc::Tile *tiles_gu, *tiles_dn;
  int* n_tiles;
  int* err;
  int max_gu, max_dn, nblk;
  size_t bytes;
};

GWs carve_gemm(void* base, int T, int K, int E, int H, int I, int r) {
  GWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off = align_up(off + n, 256);
    return base ? static_cast<char*>(base) + o : nullptr;
  };
  const size_t TK = static_cast<size_t>(T) * K, R = TK + T;
  const int rr = r > 0 ? r : 1;
  w.nblk = static_cast<int>((TK + pf::kChunk - 1) / pf::kChunk);
  const int nt_max = static_cast<int>((TK + static_cast<size_t>(E) * (gg3::BN - 1)) / gg3::BN) + (T + gg3::BN - 1) / gg3::BN + 1;
  w.max_gu = nt_max * (2 * I / gg3::BM);
  w.max_dn = nt_max * (H / gg3::BM);
  w.idx = reinterpret_cast<int32_t*>(take(TK * 4));
  w.count = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E) * 4));
  w.offset = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
  w.perm = reinterpret_cast<int32_t*>(take(TK * 4));
  w.inv = reinterpret_cast<int32_t*>(take(TK * 4));
  w.blockhist = reinterpret_cast<int32_t*>(take(static_cast<size_t>(w.nblk) * E * 4));
  w.w_pos = reinterpret_cast<float*>(take(TK * 4));
  w.t1 = reinterpret_cast<float*>(take(R * rr * 4));
  w.t2 = reinterpret_cast<float*>(take(R * rr * 4));
  w.g = reinterpret_cast<float*>(take(static_cast<size_t>(T) * 4));
  w.X = reinterpret_cast<uint16_t*>(take(R * H * 2));
  w.Hh = reinterpret_cast<uint16_t*>(take(R * I * 2));
  w.Y = reinterpret_cast<uint16_t*>(take(R * H * 2));
  w.D = reinterpret_cast<uint16_t*>(take(r > 0 ? static_cast<size_t>(T) * (2 * I > H ? 2 * I : H) * 2 : 16));
  w.tv = reinterpret_cast<float*>(take(static_cast<size_t>(T) * 2 * rr * 4));
  w.tiles_gu = reinterpret_cast<tc::Tile*>(take(static_cast<size_t>(w.max_gu) * sizeof(tc::Tile)));
  w.tiles_dn = reinterpret_cast<tc::Tile*>(take(static_cast<size_t>(w.max_dn) * sizeof(tc::Tile)));
  w.n_tiles = reinterpret_cast<int*>(take(2 * 4));
  w.err = reinterpret_cast<int*>(take(4));
  w.bytes = off;
  return w;
}

bool gemm_shapes(const moe_layer* L) {
  return L->H % gg3::BM == 0 && (2 * L->I) % gg3::BM == 0 && L->I % gg3::BK == 0;
}

// Routed gate/up adapters exist only on the tensor-core path, which serves any number of tokens.
bool gemm_path(const moe_layer* L, int T, int K) {
  return (static_cast<long long>(T) * K >= kGemmMinSlots || (L->r > 0 && L->ex_lora_A_gu)) && gemm_shapes(L);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Row-major fp16 matrix [rows][cols] as a TMA source of [32 rows x 64 cols] boxes, 128-byte swizzle.
bool token_map(CUtensorMap* m, const uint16_t* X, int cols, int rows) {
  const EncodeTiledFn f = encode_tiled();
  if (!f) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(gg3::BK), static_cast<cuuint32_t>(gg3::BROWS)};
  const cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The row records of one weight matrix in n_exp expert blocks (expert_stride bytes apart) as a 3-D byte map
// {record bytes, rows, experts}, boxes of box_x bytes x 128 rows x 1 expert (128-byte swizzle if asked).
bool weight_map(CUtensorMap* m, const uint8_t* base, int rec, int rows, int n_exp, int64_t expert_stride, int box_x,
                bool swizzle = false) {
  const EncodeTiledFn f = encode_tiled();
  if (!f) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(rec), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(n_exp)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(rec), static_cast<cuuint64_t>(expert_stride)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(gg3::BM), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor maps of one grouped GEMM over the matrix at byte a_off of every expert block (records of rec
// bytes, rows of them per expert, reduction length K).
bool gemm_maps(gg3::Maps* m, const moe_layer* L, int64_t a_off, int rec, int rows, int K, const uint16_t* tokens,
               int n_token_rows) {
  const uint8_t* pool = static_cast<const uint8_t*>(L->pool) + a_off;
  const uint8_t* sh = static_cast<const uint8_t*>(L->shared_block) + a_off;
  const int sb = gg3::sb_row_bytes(K);
  const int64_t sh_stride = static_cast<int64_t>(rec) * rows;
  return weight_map(&m->pool_codes, pool, rec, rows, L->E, L->expert_stride, 32 * gg3::RGROUPS, true) &&
         weight_map(&m->pool_sb, pool, rec, rows, L->E, L->expert_stride, sb) &&
         weight_map(&m->shared_codes, sh, rec, rows, 1, sh_stride, 32 * gg3::RGROUPS, true) &&
         weight_map(&m->shared_sb, sh, rec, rows, 1, sh_stride, sb) &&
         token_map(&m->tokens, tokens, K, n_token_rows);
}

// Row-major bf16 activations u [T][H] as a TMA source of [64 rows x 64 cols] boxes, 128-byte swizzle.
bool u_map(CUtensorMap* m, const uint16_t* u, int H, int T) {
  const EncodeTiledFn f = encode_tiled();
  if (!f) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(dense::BK), static_cast<cuuint32_t>(dense::BN)};
  const cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(u), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major matrix of `rows` rows, `cols` elements of elem_bytes each per row, row_bytes apart, as a TMA source
// of [128 rows x 128 bytes] boxes, 128-byte swizzle.
bool rows_map(CUtensorMap* m, const void* base, CUtensorMapDataType type, int elem_bytes, int cols, int rows,
              int64_t row_bytes) {
  const EncodeTiledFn f = encode_tiled();
  if (!f) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(dense::BM)};
  const cuuint32_t estr[2] = {1, 1};
  return f(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
moe_status launch_dense(const dense::Maps& m, dense::Args a, cudaStream_t st) {
  using C = dense::Cfg<MODE>;
  a.n_tiles = a.m_tiles * ((a.T + dense::BN - 1) / dense::BN);
  a.timeout_ns = kGemmTimeoutNs;
  int dev = 0, nsm = 0;
  if (cudaFuncSetAttribute(dense::dense_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
          cudaSuccess ||
      cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int grid = a.n_tiles < nsm ? a.n_tiles : nsm;
  dense::dense_kernel<MODE><<<grid, C::kThreads, C::SMEM_BYTES, st>>>(m, a);
  return launch_status();
}

bool dense_router_ok(const moe_layer* L, const uint16_t* u, int T) {
  return T >= kDenseMinTokens && L->E % dense::BM == 0 && L->router.bits == 8 && aligned(u, 16);
}

// logits [T][E] of the 8-bit router on the tensor cores.
moe_status dense_router(const moe_layer* L, const uint16_t* u, int T, float* logits, int* err, cudaStream_t st) {
  const int H = L->H, rec = qrow_bytes(H, 8);
  dense::Maps m;
  if (!u_map(&m.u, u, H, T) ||
      !rows_map(&m.a, L->router.rows, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, H, L->E, rec))
    return MOE_ERR_CUDA;
  dense::Args a{};
  a.T = T;
  a.H = H;
  a.KT = a.KTu = H / dense::BK;
  a.M = L->E;
  a.m_tiles = L->E / dense::BM;
  a.rows = static_cast<const uint8_t*>(L->router.rows);
  a.rec = rec;
  a.beta = L->router_bias;
  a.logits = logits;
  a.err = err;
  return launch_dense<dense::MODE_ROUTER>(m, a, st);
}

bool dense_w1_ok(const moe_prerouter* P, const uint16_t* u, int T) {
  return T >= kDenseMinTokens && P->P % dense::BM == 0 && P->E % dense::BK == 0 && aligned(u, 16);
}

// z [T][P] = silu(W1 [u ; multi_hot(sel)] + b1) on the tensor cores.
moe_status dense_w1(const moe_prerouter* P, const uint16_t* u, const int32_t* sel, int T, int K, float* z, int* err,
                    cudaStream_t st) {
  const int H = P->H, W = P->H + P->E;
  dense::Maps m;
  if (!u_map(&m.u, u, H, T) ||
      !rows_map(&m.a, P->W1, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, W, P->P, static_cast<int64_t>(W) * 2))
    return MOE_ERR_CUDA;
  dense::Args a{};
  a.T = T;
  a.H = H;
  a.KT = W / dense::BK;
  a.KTu = H / dense::BK;
  a.M = P->P;
  a.m_tiles = P->P / dense::BM;
  a.sel = sel;
  a.K = K;
  a.E = P->E;
  a.b1 = P->b1;
  a.z = z;
  a.err = err;
  return launch_dense<dense::MODE_W1>(m, a, st);
}

template <int H>
// Bounded waits give up after timeout_ns; drop_tile >= 0 arms the gate/up GEMM's test hook (gg3::Args).
moe_status expert_forward_gemm(const moe_layer* L, const uint16_t* u, int T, int K, const int32_t* idx, const float* w,
                               void* out, int out_mode, int32_t* perm_out, void* workspace, int* err,
                               long long timeout_ns, int drop_tile, cudaStream_t st) {
  const int E = L->E, I = L->I, TK = T * K, R = TK + T;
  // the shared expert's adapters, each projection on its own
  const bool lora_g = L->r > 0 && L->sh_lora_A[0], lora_u = L->r > 0 && L->sh_lora_A[1];
  const bool lora_d = L->r > 0 && L->sh_lora_A[2], lora_gu = lora_g || lora_u;
  const int r = L->r > 0 ? L->r : 0;
  const GWs ws = carve_gemm(workspace, T, K, E, H, I, L->r);
  int* err_dev = err ? err : ws.err;  // without a caller's word, reports go to the workspace's own (unread) word
  if (!err && cudaMemsetAsync(ws.err, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  pf::bucket_count_kernel<<<ws.nblk, pf::kChunk, 0, st>>>(idx, TK, E, ws.idx, ws.blockhist);
  pf::bucket_scan_kernel<<<1, 256, 0, st>>>(ws.nblk, E, ws.blockhist, ws.count, ws.offset);
  pf::bucket_place_kernel<<<ws.nblk, pf::kChunk, 0, st>>>(ws.idx, TK, E, ws.blockhist, ws.perm, ws.inv, perm_out);
  pf::permute_kernel<H><<<(R + 7) / 8, 256, 0, st>>>(u, T, K, ws.perm, w, ws.X, ws.w_pos, err_dev);
  pf::tile_list_kernel<<<E + 1, 128, 0, st>>>(ws.count, ws.offset, E, T, K, 2 * I / gg3::BM, H / gg3::BM, ws.tiles_gu,
                                              ws.tiles_dn, ws.n_tiles);
  // The GEMMs trust the device-built tile list: stop here if any launch so far failed.
  if (launch_status() != MOE_OK) return MOE_ERR_CUDA;
  {  // the shared expert's gate and gate/up LoRA deltas, one pass over u
    const int nt = lora_gu ? pf::shared_tokens_nt(r) : 0, smem = pf::shared_tokens_smem(H, nt);
    auto kern = nt == 0 ? pf::shared_tokens_kernel<0>
                        : (nt == 2 ? pf::shared_tokens_kernel<2> : (nt == 4 ? pf::shared_tokens_kernel<4>
                                                                            : pf::shared_tokens_kernel<8>));
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    kern<<<(T + pf::kStTok - 1) / pf::kStTok, 32 * pf::kStWarps, smem, st>>>(
        u, T, H, static_cast<const uint8_t*>(L->shared_gate.rows), ws.g, r, lora_g ? L->sh_lora_A[0] : nullptr,
        lora_u ? L->sh_lora_A[1] : nullptr, ws.tv);
    if (lora_gu)
      pf::lora_delta_kernel<<<dim3((T + pf::kStTok - 1) / pf::kStTok, (2 * I + pf::kDeltaOut - 1) / pf::kDeltaOut), 128, 0,
                              st>>>(ws.tv, T, r, true, 2 * I, lora_g ? L->sh_lora_B[0] : nullptr,
                                    lora_u ? L->sh_lora_B[1] : nullptr, L->lora_scale, ws.D);
  }
  const bool ex_gu = r > 0 && L->ex_lora_A_gu;
  if (ex_gu) {  // the routed gate/up adapters' A products on the permuted token rows
    const long long warps = static_cast<long long>(TK) * 2 * r;
    pf::lora_a_gu_rows_kernel<<<static_cast<unsigned>((warps + kWarps - 1) / kWarps), kThreads, 0, st>>>(
        ws.X, H, TK, r, L->ex_lora_A_gu, ws.idx, ws.perm, ws.t1, ws.t2);
  }
  const int RGU = qrow_bytes(H, 4), RDN = qrow_bytes(I, 4);
  const int64_t dn_off = static_cast<int64_t>(2 * I) * RGU;
  gg3::Maps m_gu, m_dn;
  if (!gemm_maps(&m_gu, L, 0, RGU, 2 * I, H, ws.X, R) || !gemm_maps(&m_dn, L, dn_off, RDN, H, I, ws.Hh, R))
    return MOE_ERR_CUDA;
  auto base_args = [&]() {
    gg3::Args a{};
    a.n_tiles = ws.n_tiles;
    a.E = E;
    a.lora_r = r;
    a.lora_scale = L->lora_scale;
    a.err = err_dev;
    a.timeout_ns = timeout_ns;
    a.drop_tile = -1;
    a.nsb = 2;
    return a;
  };
  const int smem_gu = gg3::smem_bytes(H, gg3::sb_buffers(H)), smem_dn = gg3::smem_bytes(I, gg3::sb_buffers(I));
  if (cudaFuncSetAttribute(gg3::grouped_gemm3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_gu > smem_dn ? smem_gu : smem_dn) != cudaSuccess)
    return MOE_ERR_CUDA;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  // persistent: one CTA per SM walks the tile list (the tile count is known only on the device)
  const int grid_gu = ws.max_gu < nsm ? ws.max_gu : nsm, grid_dn = ws.max_dn < nsm ? ws.max_dn : nsm;
  {  // gate/up + SwiGLU for every bucket and the shared expert
    gg3::Args a = base_args();
    a.tiles = ws.tiles_gu;
    a.K = H;
    a.nsb = gg3::sb_buffers(H);
    a.epi = tc::EPI_SWIGLU;
    a.drop_tile = drop_tile;
    a.out = ws.Hh;
    a.out_ld = I;
    if (lora_gu) {  // the shared expert's rows add their precomputed deltas
      a.lora_D = ws.D;
      a.lora_D_ld = 2 * I;
      a.lora_D_row0 = TK;
    }
    if (ex_gu) {
      a.lora_t1 = ws.t1;
      a.lora_t2 = ws.t2;
    }
    a.lora_Bgu_ex = ex_gu ? L->ex_lora_B_gu : nullptr;
    gg3::grouped_gemm3_kernel<<<grid_gu, gg3::kThreads, smem_gu, st>>>(m_gu, a);
  }
  const bool ex = r > 0 && L->ex_lora_A;
  if (lora_d) {  // the shared expert's down-projection LoRA deltas (the gate/up deltas are consumed)
    const int smem = pf::shared_down_lora_smem(I, r);
    if (cudaFuncSetAttribute(pf::shared_down_lora_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    pf::shared_down_lora_kernel<<<(T + pf::kStTok - 1) / pf::kStTok, 256, smem, st>>>(
        ws.Hh + static_cast<size_t>(TK) * I, T, I, r, L->sh_lora_A[2], ws.tv);
    pf::lora_delta_kernel<<<dim3((T + pf::kStTok - 1) / pf::kStTok, (H + pf::kDeltaOut - 1) / pf::kDeltaOut), 128, 0,
                            st>>>(ws.tv, T, r, false, H, L->sh_lora_B[2], nullptr, L->lora_scale, ws.D);
  }
  if (ex)  // the routed down adapters' A products on the SwiGLU output rows
    pf::lora_a_rows_kernel<<<(TK * r + kWarps - 1) / kWarps, kThreads, 0, st>>>(
        ws.Hh, I, TK, r, L->ex_lora_A, ws.idx, ws.perm, ws.t1);
  {  // down (+ LoRA), routed rows scaled by their gating weight
    gg3::Args a = base_args();
    a.tiles = ws.tiles_dn;
    a.n_tiles = ws.n_tiles + 1;
    a.K = I;
    a.nsb = gg3::sb_buffers(I);
    a.epi = tc::EPI_DOWN;
    a.out = ws.Y;
    a.out_ld = H;
    a.row_scale = ws.w_pos;
    if (lora_d) {
      a.lora_D = ws.D;
      a.lora_D_ld = H;
      a.lora_D_row0 = TK;
    }
    a.lora_t1 = ws.t1;
    a.lora_Bex = ex ? L->ex_lora_B : nullptr;
    gg3::grouped_gemm3_kernel<<<grid_dn, gg3::kThreads, smem_dn, st>>>(m_dn, a);
  }
  pf::combine_kernel<H><<<T, 256, 0, st>>>(ws.Y, T, K, ws.inv, ws.g, out, out_mode);
  return launch_status();
}

template <int H>
moe_status expert_forward_h(const moe_layer* L, const uint16_t* u, int T, int K, const int32_t* idx, const float* w,
                            void* out, int out_mode, int32_t* perm_out, const Ws& ws, int* err, long long timeout_ns,
                            int drop_tile, cudaStream_t st) {
  if (gemm_path(L, T, K))
    return expert_forward_gemm<H>(L, u, T, K, idx, w, out, out_mode, perm_out, ws.base, err, timeout_ns, drop_tile, st);
  if (L->r > 0 && L->ex_lora_A_gu) return MOE_ERR_UNSUPPORTED;
  switch (L->I) {
    case 128: return expert_forward_hi<H, 128>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err, st);
    case 256: return expert_forward_hi<H, 256>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err, st);
    case 512: return expert_forward_hi<H, 512>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err, st);
    case 1024: return expert_forward_hi<H, 1024>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err, st);
    case 2048: return expert_forward_hi<H, 2048>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err, st);
    default: return MOE_ERR_UNSUPPORTED;
  }
}

template <int H>
moe_status prerouter_h(const moe_prerouter* P, const uint16_t* u, const int32_t* sel, int T, int K, int K_next,
                       int32_t* pred, float* scores, float* z, int* err, cudaStream_t st) {
  if (dense_w1_ok(P, u, T)) {
    const moe_status s = dense_w1(P, u, sel, T, K, z, err, st);
    if (s != MOE_OK) return s;
  } else {
    PreW1Args a{};
    a.u = u;
    a.T = T;
    a.K = K;
    a.E = P->E;
    a.P = P->P;
    a.sel = sel;
    a.W1 = P->W1;
    a.b1 = P->b1;
    a.z = z;
    a.err = err;
    const size_t smem = gemv_smem(H, false, false);
    allow_smem(prerouter_w1_kernel<H / 8>, smem);
    dim3 g1((P->P + kWarps - 1) / kWarps, (T + TB - 1) / TB);
    prerouter_w1_kernel<H / 8><<<g1, kThreads, smem, st>>>(a);
  }
  dim3 g2((P->E_next + kW2E - 1) / kW2E, (T + kW2T - 1) / kW2T);
  prerouter_w2_kernel<<<g2, kW2Threads, 0, st>>>(z, T, P->P, P->W2, P->b2, P->E_next, scores);
  topk_kernel<<<(T + kWarps - 1) / kWarps, kThreads, 0, st>>>(scores, T, P->E_next, K_next, pred, nullptr);
  return launch_status();
}

size_t prerouter_ws(const moe_prerouter* P, int T) {
  return align_up(static_cast<size_t>(T) * P->P * 4, 256);
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA launch failed";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_RANGE: return "activation outside the fp16 range";
  }
  return "unknown status";
}

size_t moe_qrow_bytes(int32_t in_dim, int32_t bits) {
  if (in_dim <= 0 || in_dim % 64 || (bits != 4 && bits != 8)) return 0;
  return static_cast<size_t>(qrow_bytes(in_dim, bits));
}

size_t moe_expert_block_bytes(int32_t H, int32_t I) {
  if (H <= 0 || I <= 0 || H % 64 || I % 64) return 0;
  return block_bytes(H, I);
}

moe_status moe_rmsnorm_bf16(const float* x, int32_t T, int32_t H, float eps, uint16_t* u, void* stream) {
  if (T < 0 || H <= 0 || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !u) return MOE_ERR_INVALID_ARG;
  rmsnorm_bf16_kernel<<<T, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(x, H, eps, u);
  return launch_status();
}

moe_status moe_route_topk(const moe_layer* L, const uint16_t* u, int32_t T, int32_t K, float* logits, int32_t* idx,
                          float* w, int32_t* err_word, void* stream) {
  const moe_status s = check_layer(L, T, K);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!u || !logits || !idx || !w || !aligned(u, 16)) return MOE_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (L->H) {
    case 256: return route_h<256>(L, u, T, K, logits, idx, w, err_word, st);
    case 512: return route_h<512>(L, u, T, K, logits, idx, w, err_word, st);
    case 1024: return route_h<1024>(L, u, T, K, logits, idx, w, err_word, st);
    case 2048: return route_h<2048>(L, u, T, K, logits, idx, w, err_word, st);
    case 4096: return route_h<4096>(L, u, T, K, logits, idx, w, err_word, st);
    default: return MOE_ERR_UNSUPPORTED;
  }
}

static size_t ws_bytes_for(const moe_layer* L, int T, int K) {
  size_t b = carve(nullptr, T, K, L->E, L->I, L->r).bytes;
  if (gemm_path(L, T, K)) {
    const size_t g = carve_gemm(nullptr, T, K, L->E, L->H, L->I, L->r).bytes;
    if (g > b) b = g;
  }
  return b;
}

size_t moe_workspace_size(const moe_layer* L, int32_t T, int32_t K) {
  if (!L || T < 0 || T > MOE_MAX_TOKENS || K < 1) return 0;
  return ws_bytes_for(L, T, K);
}

}  // extern "C"

namespace {

// moe_expert_forward with the grouped GEMMs' wait bound and test hook exposed (the stack's per-layer path
// passes its options through).
moe_status expert_forward_entry(const moe_layer* L, const uint16_t* u, int32_t T, int32_t K, const int32_t* idx,
                                const float* w, void* out, int32_t out_mode, int32_t* perm_out, void* workspace,
                                size_t ws_bytes, int32_t* err_word, long long timeout_ns, int drop_tile,
                                void* stream) {
  moe_status s = check_layer(L, T, K);
  if (s != MOE_OK) return s;
  if (out_mode < 0 || out_mode > 2) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!u || !idx || !w || !out || !aligned(u, 16)) return MOE_ERR_INVALID_ARG;
  s = check_expert_weights(L);
  if (s != MOE_OK) return s;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_bytes_for(L, T, K)) return MOE_ERR_WORKSPACE;
  const Ws ws = carve(workspace, T, K, L->E, L->I, L->r);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (L->H) {
    case 256:
      return expert_forward_h<256>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err_word, timeout_ns, drop_tile,
                                  st);
    case 512:
      return expert_forward_h<512>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err_word, timeout_ns, drop_tile,
                                  st);
    case 1024:
      return expert_forward_h<1024>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err_word, timeout_ns, drop_tile,
                                  st);
    case 2048:
      return expert_forward_h<2048>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err_word, timeout_ns, drop_tile,
                                  st);
    case 4096:
      return expert_forward_h<4096>(L, u, T, K, idx, w, out, out_mode, perm_out, ws, err_word, timeout_ns, drop_tile,
                                  st);
    default: return MOE_ERR_UNSUPPORTED;
  }
}

}  // namespace

extern "C" {

moe_status moe_expert_forward(const moe_layer* L, const uint16_t* u, int32_t T, int32_t K, const int32_t* idx,
                              const float* w, void* out, int32_t out_mode, int32_t* perm_out, void* workspace,
                              size_t ws_bytes, int32_t* err_word, void* stream) {
  return expert_forward_entry(L, u, T, K, idx, w, out, out_mode, perm_out, workspace, ws_bytes, err_word,
                              kGemmTimeoutNs, -1, stream);
}

size_t prerouter_workspace_size(const moe_prerouter* head, int32_t T) {
  if (!head || T < 0 || T > MOE_MAX_TOKENS) return 0;
  return prerouter_ws(head, T);
}

moe_status prerouter_predict(const moe_prerouter* head, const uint16_t* u, const int32_t* sel, int32_t T, int32_t K,
                             int32_t K_next, int32_t* pred, float* scores, void* workspace, size_t ws_bytes,
                             int32_t* err_word, void* stream) {
  if (!head) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > MOE_MAX_TOKENS) return MOE_ERR_UNSUPPORTED;
  moe_status s = check_head_shape(head, K, K_next);
  if (s != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!u || !sel || !pred || !scores || !aligned(u, 16)) return MOE_ERR_INVALID_ARG;
  s = check_head_weights(head);
  if (s != MOE_OK) return s;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < prerouter_ws(head, T)) return MOE_ERR_WORKSPACE;
  float* z = static_cast<float*>(workspace);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (head->H) {
    case 256: return prerouter_h<256>(head, u, sel, T, K, K_next, pred, scores, z, err_word, st);
    case 512: return prerouter_h<512>(head, u, sel, T, K, K_next, pred, scores, z, err_word, st);
    case 1024: return prerouter_h<1024>(head, u, sel, T, K, K_next, pred, scores, z, err_word, st);
    case 2048: return prerouter_h<2048>(head, u, sel, T, K, K_next, pred, scores, z, err_word, st);
    case 4096: return prerouter_h<4096>(head, u, sel, T, K, K_next, pred, scores, z, err_word, st);
    default: return MOE_ERR_UNSUPPORTED;
  }
}


}  // extern "C"

// ----------------------------------------------------------------------------- stacked decode
namespace {

inline uint32_t al128(size_t x) { return static_cast<uint32_t>(align_up(x, 128)); }

// Layout and eligibility of the persistent single-launch path.
struct Persist {
  bool ok = false;
  stk::Smem sm{};
  int NA = 0, grid = 0;
  int ll_x = 0, ll_a = 0, ll_h = 0, ll_z = 0, ll_p = 0, ll_stride = 0;
  size_t ll_bytes = 0;
};

Persist plan_persistent(const moe_layer* Ls, const moe_prerouter* Ps, int n, int T, int K, int K_next, int use_pred) {
  Persist pl;
  const moe_layer& L0 = Ls[0];
  const int H = L0.H, E = L0.E, I = L0.I, r = L0.r;
  if (T != 1 || use_pred || n > stk::kMaxLayers || (H != 1024 && H != 2048) || I != 512 || E % 8) return pl;
  const bool lora = r > 0 && L0.sh_lora_A[0];
  if (lora && (r % 8 || r > 32)) return pl;
  for (int l = 0; l < n; ++l) {
    const moe_layer& L = Ls[l];
    if (L.ex_lora_A || L.ex_lora_A_gu) return pl;
    for (int q = 0; q < 3; ++q)
      if ((L.sh_lora_A[q] != nullptr) != lora || (L.sh_lora_B[q] != nullptr) != lora) return pl;
    if (!L.shared_block || !aligned(L.shared_block, 16) || !qrows_ok(L.shared_gate, 1, H, 8)) return pl;
    if (!L.pool || !aligned(L.pool, 256) || L.expert_stride != L0.expert_stride || L.expert_stride % 256) return pl;
    if (Ps && (!Ps[l].W1 || !Ps[l].b1 || !Ps[l].W2 || !Ps[l].b2 || !aligned(Ps[l].W1, 16) || !aligned(Ps[l].W2, 16)))
      return pl;
  }
  const int P = Ps ? Ps[0].P : 0, En = Ps ? Ps[0].E_next : 0;
  if (Ps && (P % 8 || P > 2048 || En > 256 || En < K || K_next != K)) return pl;
  int dev = 0, nsm = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || nsm <= 0)
    return pl;
  const int N = nsm;
  const int NA = E + 1 + (lora ? 2 * r : 0);
  auto cdiv = [](int a, int b) { return (a + b - 1) / b; };
  stk::Smem& S = pl.sm;
  S.maxA = cdiv(NA, N);
  S.maxS = cdiv(I / 2, N);
  S.maxR = cdiv(K * I / 2, N);
  S.maxD = cdiv(H, N);
  S.maxZ = P ? cdiv(P, N) : 0;
  S.maxP = En ? cdiv(En, N) : 0;
  const int RGU = qrow_bytes(H, 4), RDN = qrow_bytes(I, 4), R8 = qrow_bytes(H, 8), UNIT = 4 * RGU;
  S.item_bytes = static_cast<int>(align_up(static_cast<size_t>(R8 > 2 * H ? R8 : 2 * H), 16));
  size_t o = 0;
  auto put = [&](size_t bytes) {
    const uint32_t at = al128(o);
    o = at + bytes;
    return at;
  };
  S.o_items = put(static_cast<size_t>(S.maxA) * S.item_bytes);
  S.o_shu = put(static_cast<size_t>(S.maxS) * UNIT);
  S.o_shB = put(static_cast<size_t>(S.maxS) * 8 * r);
  S.o_sdn = put(static_cast<size_t>(S.maxD) * RDN);
  S.o_Bd = put(static_cast<size_t>(S.maxD) * 2 * r);
  S.o_Ad = put(static_cast<size_t>(r) * I * 2);
  S.o_W1 = put(static_cast<size_t>(S.maxZ) * 2 * H);
  const uint32_t st_bytes = al128(o);
  o = 0;
  S.st[0] = put(st_bytes);
  S.st[1] = put(st_bytes);
  S.units = put(static_cast<size_t>(S.maxR) * UNIT);
  S.down = put(static_cast<size_t>(K) * S.maxD * RDN);
  S.xs = put(4 * H);
  S.un = put(2 * H);
  S.up = put(2 * H);
  S.s16 = put(4 * H / 16);
  S.s32 = put(4 * H / 32);
  S.hs = put(2 * (K + 1) * I);
  S.hsum = put(4 * (K + 1) * I / 32);
  S.hraw = put(4 * (K + 1) * I / 2);
  S.logit = put(4 * ((E > En ? E : En) + 1 + 2 * r));
  S.td = put(4 * (r + 1));
  S.yd = put(4 * S.maxD * (K + 1));
  S.red = put(4 * 64);
  S.z = put(4 * (P + 1));
  S.hloc = put(4 * 2 * (S.maxS + S.maxR));
  S.bar = put(8 * (3 + S.maxR));
  S.sent = put(4 * 6 * N);
  S.total = al128(o);
  if (static_cast<int>(S.total) > optin) return pl;
  pl.NA = NA;
  pl.ll_x = 0;
  pl.ll_a = H;
  pl.ll_h = pl.ll_a + NA;
  pl.ll_z = pl.ll_h + (K + 1) * I / 2;
  pl.ll_stride = (pl.ll_z + P + 31) / 32 * 32;
  pl.ll_p = 2 * pl.ll_stride;
  pl.ll_bytes = (static_cast<size_t>(pl.ll_p) + static_cast<size_t>(n) * En) * 8;
  pl.grid = N;
  pl.ok = true;
  return pl;
}

template <int H>
cudaError_t launch_persistent(const Persist& pl, const moe_layer* Ls, const moe_prerouter* Ps, int n, int K, float eps,
                              float* x, float* x_trace, uint16_t* u_trace, int32_t* idx_all, int32_t* true_idx_all,
                              int32_t* pred_all, int32_t* err, unsigned long long* ll, const moe_stack_opts* opts,
                              cudaStream_t st) {
  auto kern = stk::stack_decode_kernel<H, 512>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.sm.total));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, stk::kThreads, pl.sm.total);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  stk::Params p{};
  const moe_layer& L0 = Ls[0];
  p.n_layers = n;
  p.E = L0.E;
  p.K = K;
  p.r = (L0.r > 0 && L0.sh_lora_A[0]) ? L0.r : 0;
  p.P = Ps ? Ps[0].P : 0;
  p.En = Ps ? Ps[0].E_next : 0;
  p.NA = pl.NA;
  p.stride = L0.expert_stride;
  p.eps = eps;
  p.lora_scale = L0.lora_scale;
  p.x = x;
  p.x_trace = x_trace;
  p.u_trace = u_trace;
  p.idx_all = idx_all;
  p.true_idx_all = true_idx_all;
  p.pred_all = pred_all;
  p.err = err;
  p.ll = ll;
  p.ll_x = pl.ll_x;
  p.ll_a = pl.ll_a;
  p.ll_h = pl.ll_h;
  p.ll_z = pl.ll_z;
  p.ll_p = pl.ll_p;
  p.ll_stride = pl.ll_stride;
  p.timeout_ns = (opts && opts->timeout_ns > 0) ? opts->timeout_ns : 1000000000LL;
  p.drop_layer = (opts && opts->test_drop_layer > 0) ? opts->test_drop_layer - 1 : -1;
  p.drop_cta = opts ? opts->test_drop_cta : -1;
  p.trace = opts ? reinterpret_cast<long long*>(opts->trace) : nullptr;
  p.sm = pl.sm;
  for (int l = 0; l < n; ++l) {
    const moe_layer& L = Ls[l];
    stk::LayerPtrs& d = p.L[l];
    d.router = static_cast<const uint8_t*>(L.router.rows);
    d.rbias = L.router_bias;
    d.sgate = static_cast<const uint8_t*>(L.shared_gate.rows);
    d.shared = static_cast<const uint8_t*>(L.shared_block);
    if (p.r) {
      d.Ag = L.sh_lora_A[0];
      d.Bg = L.sh_lora_B[0];
      d.Au = L.sh_lora_A[1];
      d.Bu = L.sh_lora_B[1];
      d.Ad = L.sh_lora_A[2];
      d.Bd = L.sh_lora_B[2];
    }
    d.pool = static_cast<const uint8_t*>(L.pool);
    if (Ps) {
      d.W1 = Ps[l].W1;
      d.b1 = Ps[l].b1;
      d.W2 = Ps[l].W2;
      d.b2 = Ps[l].b2;
    }
  }
  void* args[] = {&p};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(pl.grid), dim3(stk::kThreads), args,
                                    pl.sm.total, st);
}

// Layout of the second-generation single-launch kernel (same eligibility as plan_persistent).
struct Persist2 {
  bool ok = false;
  stk2::Smem sm{};
  int NA = 0, grid = 0;
  int ll_x = 0, ll_a = 0, ll_h = 0, ll_z = 0, ll_p = 0, ll_stride = 0, st_bytes = 0;
  size_t ll_bytes = 0;
};

Persist2 plan_persistent2(const moe_layer* Ls, const moe_prerouter* Ps, int n, int T, int K, int K_next, int use_pred) {
  Persist2 pl;
  const moe_layer& L0 = Ls[0];
  const int H = L0.H, E = L0.E, I = L0.I, r = L0.r;
  if (T != 1 || use_pred || n > stk::kMaxLayers || (H != 1024 && H != 2048) || I != 512 || E % 8 || K > stk2::kMaxK)
    return pl;
  const bool lora = r > 0 && L0.sh_lora_A[0];
  if (lora && (r % 8 || r > 32)) return pl;
  for (int l = 0; l < n; ++l) {
    const moe_layer& L = Ls[l];
    if (L.ex_lora_A || L.ex_lora_A_gu) return pl;
    for (int q = 0; q < 3; ++q)
      if ((L.sh_lora_A[q] != nullptr) != lora || (L.sh_lora_B[q] != nullptr) != lora) return pl;
    if (!L.shared_block || !aligned(L.shared_block, 16) || !qrows_ok(L.shared_gate, 1, H, 8)) return pl;
    if (!L.pool || !aligned(L.pool, 256) || L.expert_stride != L0.expert_stride || L.expert_stride % 256) return pl;
    if (Ps && (!Ps[l].W1 || !Ps[l].b1 || !Ps[l].W2 || !Ps[l].b2 || !aligned(Ps[l].W1, 16) || !aligned(Ps[l].W2, 16)))
      return pl;
  }
  const int P = Ps ? Ps[0].P : 0, En = Ps ? Ps[0].E_next : 0;
  if (Ps && (P % 8 || P > 2048 || En > 256 || En < K || K_next != K)) return pl;
  int dev = 0, nsm = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || nsm <= 0)
    return pl;
  const int N = nsm;
  const int NA = E + 1 + (lora ? 2 * r : 0);
  auto cdiv = [](int a, int b) { return (a + b - 1) / b; };
  stk2::Smem& S = pl.sm;
  S.maxA = cdiv(NA, N);
  S.maxS = cdiv(I / 2, N);
  S.maxR = cdiv(K * I / 2, N);
  S.maxD = cdiv(H, N);
  S.maxZ = P ? cdiv(P, N) : 0;
  // per-thread roles of the kernel: SwiGLU words by threads < 480, Prerouter words by the last warp's
  // lanes, 16 combine lanes per output row
  if (S.maxS + S.maxR > stk2::kThreads - 32 || S.maxZ > 32 || S.maxD > 2 * stk2::kWarps) return pl;
  const int RGU = qrow_bytes(H, 4), RDN = qrow_bytes(I, 4), R8 = qrow_bytes(H, 8), UNIT = 4 * RGU;
  S.item_bytes = static_cast<int>(align_up(static_cast<size_t>(R8 > 2 * H ? R8 : 2 * H), 16));
  size_t o = 0;
  auto put = [&](size_t bytes) {
    const uint32_t at = al128(o);
    o = at + bytes;
    return at;
  };
  S.o_items = put(static_cast<size_t>(S.maxA) * S.item_bytes);
  S.o_shu = put(static_cast<size_t>(S.maxS) * UNIT);
  S.o_shB = put(static_cast<size_t>(S.maxS) * 8 * r);
  S.o_sdn = put(static_cast<size_t>(S.maxD) * RDN);
  S.o_Bd = put(static_cast<size_t>(S.maxD) * 2 * r);
  S.o_Ad = put(static_cast<size_t>(r) * I * 2);
  S.o_W1 = put(static_cast<size_t>(S.maxZ) * 2 * H);
  const uint32_t st_bytes = al128(o);
  o = 0;
  S.st[0] = put(st_bytes);
  S.st[1] = put(st_bytes);
  S.units = put(static_cast<size_t>(S.maxR) * UNIT);
  S.down = put(static_cast<size_t>(K) * S.maxD * RDN);
  S.xs = put(4 * H);
  S.un = put(2 * H);
  S.up = put(2 * H);
  S.s16 = put(4 * H / 16);
  S.s32 = put(4 * H / 32);
  S.hs = put(2 * (K + 1) * I);
  S.hsum = put(4 * (K + 1) * I / 32);
  S.logit = put(4 * ((E > En ? E : En) + 1 + 2 * r));
  S.td = put(4 * (r + 1));
  S.yd = put(4 * S.maxD * (K + 1));
  S.red = put(4 * 64);
  S.zx = put(4 * (S.maxZ + 1));
  S.hloc = put(4 * 2 * (S.maxS + S.maxR));
  S.shacc = put(4 * 4 * (S.maxS + 1));
  S.bar = put(8 * (2 + S.maxR + stk2::kMaxK));
  S.total = al128(o);
  if (static_cast<int>(S.total) > optin) return pl;
  pl.NA = NA;
  pl.ll_x = 0;
  pl.ll_a = H;
  pl.ll_h = pl.ll_a + NA;
  pl.ll_stride = (pl.ll_h + (K + 1) * I / 2 + 31) / 32 * 32;
  pl.ll_z = 2 * pl.ll_stride;
  pl.ll_p = pl.ll_z + n * P;
  pl.ll_bytes = (static_cast<size_t>(pl.ll_p) + static_cast<size_t>(n) * En) * 8;
  pl.st_bytes = static_cast<int>(st_bytes);
  pl.grid = N;
  pl.ok = true;
  return pl;
}

template <int H>
cudaError_t launch_persistent2(const Persist2& pl, const moe_layer* Ls, const moe_prerouter* Ps, int n, int K,
                               float eps, float* x, float* x_trace, uint16_t* u_trace, int32_t* idx_all,
                               int32_t* true_idx_all, int32_t* pred_all, int32_t* err, unsigned long long* ll,
                               const moe_stack_opts* opts, cudaStream_t st) {
  auto kern = stk2::stack_decode2_kernel<H, 512>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.sm.total));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, stk2::kThreads, pl.sm.total);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  stk2::Params p{};
  const moe_layer& L0 = Ls[0];
  p.n_layers = n;
  p.E = L0.E;
  p.K = K;
  p.r = (L0.r > 0 && L0.sh_lora_A[0]) ? L0.r : 0;
  p.P = Ps ? Ps[0].P : 0;
  p.En = Ps ? Ps[0].E_next : 0;
  p.NA = pl.NA;
  p.stride = L0.expert_stride;
  p.eps = eps;
  p.lora_scale = L0.lora_scale;
  p.x = x;
  p.x_trace = x_trace;
  p.u_trace = u_trace;
  p.idx_all = idx_all;
  p.true_idx_all = true_idx_all;
  p.pred_all = pred_all;
  p.err = err;
  p.ll = ll;
  p.ll_x = pl.ll_x;
  p.ll_a = pl.ll_a;
  p.ll_h = pl.ll_h;
  p.ll_z = pl.ll_z;
  p.ll_p = pl.ll_p;
  p.ll_stride = pl.ll_stride;
  p.st_bytes = pl.st_bytes;
  p.timeout_ns = (opts && opts->timeout_ns > 0) ? opts->timeout_ns : 1000000000LL;
  p.drop_layer = (opts && opts->test_drop_layer > 0) ? opts->test_drop_layer - 1 : -1;
  p.drop_cta = opts ? opts->test_drop_cta : -1;
  p.trace = opts ? reinterpret_cast<long long*>(opts->trace) : nullptr;
  p.sm = pl.sm;
  for (int l = 0; l < n; ++l) {
    const moe_layer& L = Ls[l];
    stk::LayerPtrs& d = p.L[l];
    d.router = static_cast<const uint8_t*>(L.router.rows);
    d.rbias = L.router_bias;
    d.sgate = static_cast<const uint8_t*>(L.shared_gate.rows);
    d.shared = static_cast<const uint8_t*>(L.shared_block);
    if (p.r) {
      d.Ag = L.sh_lora_A[0];
      d.Bg = L.sh_lora_B[0];
      d.Au = L.sh_lora_A[1];
      d.Bu = L.sh_lora_B[1];
      d.Ad = L.sh_lora_A[2];
      d.Bd = L.sh_lora_B[2];
    }
    d.pool = static_cast<const uint8_t*>(L.pool);
    if (Ps) {
      d.W1 = Ps[l].W1;
      d.b1 = Ps[l].b1;
      d.W2 = Ps[l].W2;
      d.b2 = Ps[l].b2;
    }
  }
  void* args[] = {&p};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(pl.grid), dim3(stk2::kThreads), args,
                                    pl.sm.total, st);
}

struct StackWs {
  uint16_t* u;
  float *logits, *w, *scores;
  int32_t *idx_true, *pred0, *pred1, *err;
  unsigned long long* ll;
  void* ews;
  size_t ews_bytes;
  void* pws;
  size_t pws_bytes;
  size_t bytes;
};

StackWs carve_stack(void* base, const moe_layer* L0, const moe_prerouter* P0, int T, int K, int K_next, size_t ll_bytes) {
  StackWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off = align_up(off + n, 256);
    return base ? static_cast<char*>(base) + o : nullptr;
  };
  const int E_next = P0 ? P0->E_next : 1;
  w.u = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(T) * L0->H * 2));
  w.logits = reinterpret_cast<float*>(take(static_cast<size_t>(T) * L0->E * 4));
  w.w = reinterpret_cast<float*>(take(static_cast<size_t>(T) * K * 4));
  w.scores = reinterpret_cast<float*>(take(static_cast<size_t>(T) * E_next * 4));
  w.idx_true = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * K * 4));
  w.pred0 = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * K_next * 4));
  w.pred1 = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * K_next * 4));
  w.err = reinterpret_cast<int32_t*>(take(4));
  w.ll = reinterpret_cast<unsigned long long*>(take(ll_bytes));
  w.ews_bytes = ws_bytes_for(L0, T, K);
  w.ews = take(w.ews_bytes);
  w.pws_bytes = P0 ? prerouter_ws(P0, T) : 0;
  w.pws = take(w.pws_bytes);
  w.bytes = off;
  return w;
}

// Upper bound of the epoch-word region (two parity halves + one Prerouter hidden and score vector per layer).
size_t ll_bound(const moe_layer* L0, const moe_prerouter* P0, int K, int n_layers) {
  const int NA = L0->E + 1 + 2 * (L0->r > 0 ? L0->r : 0);
  const size_t words = L0->H + NA + static_cast<size_t>(K + 1) * L0->I / 2 + (P0 ? P0->P : 0) + 32;
  return (2 * words + static_cast<size_t>(n_layers) * (P0 ? P0->E_next + P0->P : 0)) * 8;
}

}  // namespace

extern "C" {

int32_t moe_stack_grid(void) {
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return nsm;
}

size_t moe_stack_workspace_size(const moe_layer* layers, const moe_prerouter* heads, int32_t n_layers, int32_t T,
                                int32_t K, int32_t K_next) {
  if (!layers || n_layers < 1 || T < 0 || T > MOE_MAX_TOKENS || K < 1) return 0;
  return carve_stack(nullptr, &layers[0], heads, T, K, K_next, ll_bound(&layers[0], heads, K, n_layers)).bytes;
}

moe_status moe_stack_decode(const moe_layer* layers, const moe_prerouter* heads, int32_t n_layers, int32_t T,
                            int32_t K, int32_t K_next, float eps, float* x, float* x_trace, uint16_t* u_trace,
                            int32_t* idx_all, int32_t* true_idx_all, int32_t* pred_all, int32_t use_predicted_routing,
                            int32_t* err_word, const moe_stack_opts* opts, void* workspace, size_t ws_bytes,
                            void* stream) {
  if (!layers || n_layers < 1 || !x) return MOE_ERR_INVALID_ARG;
  if (use_predicted_routing && (!heads || K_next != K)) return MOE_ERR_INVALID_ARG;
  if (opts && (opts->path < 0 || opts->path > 3)) return MOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    const moe_status s = check_layer(&layers[l], T, K);
    if (s != MOE_OK) return s;
    if (layers[l].H != layers[0].H || layers[l].E != layers[0].E || layers[l].I != layers[0].I ||
        layers[l].r != layers[0].r)
      return MOE_ERR_UNSUPPORTED;
    if (heads && (heads[l].H != layers[0].H || heads[l].E != layers[0].E || heads[l].E_next != heads[0].E_next ||
                  heads[l].P != heads[0].P))
      return MOE_ERR_UNSUPPORTED;
    if (heads) {
      const moe_status hs = check_head_shape(&heads[l], K, K_next);
      if (hs != MOE_OK) return hs;
    }
  }
  if (T == 0) return MOE_OK;
  // Every layer's weights are checked here, so that no launch happens for a stack that would fail part-way.
  for (int l = 0; l < n_layers; ++l) {
    moe_status s = check_expert_weights(&layers[l]);
    if (s == MOE_OK && heads) s = check_head_weights(&heads[l]);
    if (s != MOE_OK) return s;
  }
  const size_t llb = ll_bound(&layers[0], heads, K, n_layers);
  const StackWs need = carve_stack(nullptr, &layers[0], heads, T, K, K_next, llb);
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < need.bytes) return MOE_ERR_WORKSPACE;
  const StackWs ws = carve_stack(workspace, &layers[0], heads, T, K, K_next, llb);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = layers[0].H, E = layers[0].E;
  int32_t* err = err_word ? err_word : ws.err;
  if (cudaMemsetAsync(err, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;

  const int want = opts ? opts->path : 0;
  if (want == 0 || want == 2) {
    const Persist2 pl = plan_persistent2(layers, heads, n_layers, T, K, K_next, use_predicted_routing);
    if (pl.ok && pl.ll_bytes <= llb) {
      if (cudaMemsetAsync(ws.ll, 0, pl.ll_bytes, st) != cudaSuccess) return MOE_ERR_CUDA;
      const cudaError_t e =
          H == 2048 ? launch_persistent2<2048>(pl, layers, heads, n_layers, K, eps, x, x_trace, u_trace, idx_all,
                                               true_idx_all, pred_all, err, ws.ll, opts, st)
                    : launch_persistent2<1024>(pl, layers, heads, n_layers, K, eps, x, x_trace, u_trace, idx_all,
                                               true_idx_all, pred_all, err, ws.ll, opts, st);
      return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
    if (want == 2) return MOE_ERR_UNSUPPORTED;
  }
  if (want == 3) {
    const Persist pl = plan_persistent(layers, heads, n_layers, T, K, K_next, use_predicted_routing);
    if (!pl.ok || pl.ll_bytes > llb) return MOE_ERR_UNSUPPORTED;
    if (cudaMemsetAsync(ws.ll, 0, pl.ll_bytes, st) != cudaSuccess) return MOE_ERR_CUDA;
    const cudaError_t e =
        H == 2048 ? launch_persistent<2048>(pl, layers, heads, n_layers, K, eps, x, x_trace, u_trace, idx_all,
                                            true_idx_all, pred_all, err, ws.ll, opts, st)
                  : launch_persistent<1024>(pl, layers, heads, n_layers, K, eps, x, x_trace, u_trace, idx_all,
                                            true_idx_all, pred_all, err, ws.ll, opts, st);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }

  const size_t TK = static_cast<size_t>(T) * K, TKn = static_cast<size_t>(T) * K_next;
  int32_t* pred_prev = nullptr;
  for (int l = 0; l < n_layers; ++l) {
    const moe_layer* L = &layers[l];
    uint16_t* u = u_trace ? u_trace + static_cast<size_t>(l) * T * H : ws.u;
    if (x_trace && cudaMemcpyAsync(x_trace + static_cast<size_t>(l) * T * H, x, static_cast<size_t>(T) * H * 4,
                                   cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    moe_status s = moe_rmsnorm_bf16(x, T, H, eps, u, stream);
    if (s != MOE_OK) return s;
    int32_t* idx_true = true_idx_all ? true_idx_all + l * TK : (idx_all && !use_predicted_routing ? idx_all + l * TK
                                                                                                    : ws.idx_true);
    s = moe_route_topk(L, u, T, K, ws.logits, idx_true, ws.w, err, stream);
    if (s != MOE_OK) return s;
    const int32_t* idx_exec = idx_true;
    if (use_predicted_routing && l > 0) {
      gate_at_kernel<<<(T + kWarps - 1) / kWarps, kThreads, 0, st>>>(ws.logits, T, E, K, pred_prev, ws.w);
      idx_exec = pred_prev;
    }
    if (idx_all && idx_all + l * TK != idx_exec &&
        cudaMemcpyAsync(idx_all + l * TK, idx_exec, TK * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    const long long gemm_to = (opts && opts->timeout_ns > 0) ? opts->timeout_ns : kGemmTimeoutNs;
    const int drop = (opts && opts->test_drop_layer == l + 1) ? opts->test_drop_cta : -1;
    s = expert_forward_entry(L, u, T, K, idx_exec, ws.w, x, 2, nullptr, ws.ews, ws.ews_bytes, err, gemm_to, drop,
                             stream);
    if (s != MOE_OK) return s;
    if (heads) {
      int32_t* pred = pred_all ? pred_all + l * TKn : ((l & 1) ? ws.pred1 : ws.pred0);
      s = prerouter_predict(&heads[l], u, idx_exec, T, K, K_next, pred, ws.scores, ws.pws, ws.pws_bytes, err, stream);
      if (s != MOE_OK) return s;
      pred_prev = pred;
    }
  }
  return launch_status();
}

}  // extern "C"

// ----------------------------------------------------------------------------- allocation-free variant
// Scratch for moe_expert_forward_noalloc lives in this fixed device array
// instead of a caller-provided workspace.  Every GPU that loads the library
// reserves it until the process exits.  In host code the name is only a
// host-side stand-in: its device address is fetched once per device with
// cudaGetSymbolAddress and passed to the kernels.
namespace {

constexpr size_t kStaticScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device, looked up on first use.  A failed lookup is
// not remembered: the next call tries again.
moe_status static_scratch(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();  // leave no sticky launch status behind
      return MOE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

moe_status moe_expert_forward_noalloc(const moe_layer* L, const uint16_t* u, int32_t T, int32_t K,
                                      const int32_t* idx, const float* w, void* out, int32_t out_mode,
                                      int32_t* perm_out, int32_t* err_word, void* stream) {
  moe_status s = check_layer(L, T, K);
  if (s != MOE_OK) return s;
  if (out_mode < 0 || out_mode > 2) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (moe_workspace_size(L, T, K) > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = static_scratch(&scratch);
  if (s != MOE_OK) return s;
  return moe_expert_forward(L, u, T, K, idx, w, out, out_mode, perm_out, scratch, kStaticScratchBytes, err_word,
                            stream);
}

}  // extern "C"


// ----------------------------------------------------------------------------- tiered expert pool
struct moe_tier : moe::tier::Tier {};

extern "C" {

moe_status moe_tier_create(const void* host_pool, int64_t host_stride, int32_t n_experts, int64_t block_bytes,
                           void* hbm_slots, int64_t slot_stride, int32_t n_slots, moe_tier** out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!host_pool || !hbm_slots || n_experts < 1 || n_experts > moe::tier::kMaxExperts || n_slots < 1 ||
      block_bytes < 1 || host_stride < block_bytes || slot_stride < block_bytes || slot_stride % 256 != 0 ||
      !aligned(hbm_slots, 256))
    return MOE_ERR_INVALID_ARG;
  cudaPointerAttributes ah{}, ad{};
  if (cudaPointerGetAttributes(&ah, host_pool) != cudaSuccess || ah.type != cudaMemoryTypeHost ||
      cudaPointerGetAttributes(&ad, hbm_slots) != cudaSuccess || ad.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return MOE_ERR_INVALID_ARG;
  }
  moe_tier* t = new moe_tier();
  t->host = static_cast<const uint8_t*>(host_pool);
  t->host_stride = host_stride;
  t->E = n_experts;
  t->bytes = block_bytes;
  t->slots = static_cast<uint8_t*>(hbm_slots);
  t->slot_stride = slot_stride;
  t->S = n_slots;
  t->slot_of.assign(n_experts, -1);
  t->expert_in.assign(n_slots, -1);
  t->last_use.assign(n_slots, 0);
  t->prefetched.assign(n_slots, 0);
  if (cudaEventCreateWithFlags(&t->use_ev, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&t->pf_ev, cudaEventDisableTiming) != cudaSuccess) {
    if (t->use_ev) cudaEventDestroy(t->use_ev);
    delete t;
    return MOE_ERR_CUDA;
  }
  *out = t;
  return MOE_OK;
}

void moe_tier_destroy(moe_tier* t) {
  if (!t) return;
  cudaEventDestroy(t->use_ev);
  cudaEventDestroy(t->pf_ev);
  delete t;
}

moe_status moe_tier_acquire(moe_tier* t, const int32_t* experts, int32_t n_list, const int32_t* idx,
                            int32_t n_idx, int32_t* idx_slot, int32_t* err_word, void* stream) {
  if (!t || (n_list > 0 && !experts) || n_list < 0 || n_idx < 0 || (n_idx > 0 && (!idx || !idx_slot)))
    return MOE_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(t->mu);
  const std::vector<int32_t> want = t->distinct(experts, n_list);
  if (static_cast<int>(want.size()) > t->S) return MOE_ERR_WORKSPACE;
  if (t->pf_pending) {  // the prefetched blocks are complete before anything later on this stream
    if (cudaStreamWaitEvent(st, t->pf_ev, 0) != cudaSuccess) return MOE_ERR_CUDA;
    t->pf_pending = false;
  }
  ++t->tick;
  std::vector<int32_t> missing;
  for (int e : want) {
    const int s = t->slot_of[e];
    if (s >= 0) {
      ++t->st.hits;
      if (t->prefetched[s]) ++t->st.prefetch_hits;
      t->prefetched[s] = 0;
      t->last_use[s] = t->tick;
    } else {
      missing.push_back(e);
    }
  }
  t->acq_tick = t->tick;
  for (int e : missing) {  // no slot wanted at this tick is reused: the call's experts stay resident
    const int v = t->victim(t->tick);
    if (v < 0) return MOE_ERR_WORKSPACE;
    if (!t->place(e, v, st)) return MOE_ERR_CUDA;
    t->prefetched[v] = 0;
    ++t->st.misses;
    t->st.bytes_acquired += t->bytes;
  }
  ++t->st.acquires;
  t->st.requested += static_cast<int64_t>(want.size());
  if (n_idx > 0) {
    moe::tier::Table tab;
    for (int e = 0; e < moe::tier::kMaxExperts; ++e) tab.slot[e] = e < t->E ? t->slot_of[e] : -1;
    const int threads = 256, blocks = (n_idx + threads - 1) / threads;
    moe::tier::remap_kernel<<<blocks < 1024 ? blocks : 1024, threads, 0, st>>>(idx, n_idx, tab, t->E, idx_slot,
                                                                                 err_word);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

moe_status moe_tier_release(moe_tier* t, void* stream) {
  if (!t) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(t->mu);
  if (cudaEventRecord(t->use_ev, static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  t->use_recorded = true;
  return MOE_OK;
}

moe_status moe_tier_prefetch(moe_tier* t, const int32_t* experts, int32_t n, void* copy_stream) {
  if (!t || n < 0 || (n > 0 && !experts)) return MOE_ERR_INVALID_ARG;
  const cudaStream_t cs = static_cast<cudaStream_t>(copy_stream);
  std::lock_guard<std::mutex> lock(t->mu);
  std::vector<int32_t> want = t->distinct(experts, n);
  if (static_cast<int>(want.size()) > t->S) want.resize(t->S);
  // no copy may overwrite a slot before the kernels enqueued up to the last release have read it
  if (t->use_recorded && cudaStreamWaitEvent(cs, t->use_ev, 0) != cudaSuccess) return MOE_ERR_CUDA;
  ++t->tick;
  for (int e : want)
    if (t->slot_of[e] >= 0) t->last_use[t->slot_of[e]] = t->tick;
  bool any = false;
  for (int e : want) {
    if (t->slot_of[e] >= 0) continue;
    const int v = t->victim(t->acq_tick);  // the last acquire's experts are never evicted by a prefetch
    if (v < 0) break;
    if (!t->place(e, v, cs)) return MOE_ERR_CUDA;
    t->prefetched[v] = 1;
    ++t->st.prefetched;
    t->st.bytes_prefetched += t->bytes;
    any = true;
  }
  if (any || t->pf_pending) {
    if (cudaEventRecord(t->pf_ev, cs) != cudaSuccess) return MOE_ERR_CUDA;
    t->pf_pending = true;
  }
  return MOE_OK;
}

moe_status moe_tier_get_stats(const moe_tier* t, moe_tier_stats* out) {
  if (!t || !out) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(const_cast<moe_tier*>(t)->mu);
  *out = t->st;
  return MOE_OK;
}

}  // extern "C"
