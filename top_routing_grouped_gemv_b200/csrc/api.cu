// C ABI of the MoE layer forward (include/moe.h): the two-phase interface of
// aclnnQuantGroupedMatMulAlltoAllv (return-value section: phase 1 validates
// the parameters and sizes the workspace and the executor, phase 2 runs),
// argument validation against that page's constraints, the workspace layout
// and the launch sequence of each stage.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "moe.h"
#include "kernels.h"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

constexpr int kMaxEvents = 16;
// host-buffer path events: per staging slot s: in_done[s], out_ready[s], slot_free[s]
constexpr int kHostEvents = 6;

struct Layout {
  size_t status = 0, counter = 0, chunk_counts = 0, h = 0, h_end = 0;
  size_t ids = 0, gates = 0, pos = 0, src = 0, slot = 0, counts = 0, offsets = 0, x_perm = 0,
         y_perm = 0, tok_scale = 0, simt_part = 0;
  size_t fwd_end = 0, x_stage = 0, y_stage = 0, total = 0, x_stage_bytes = 0, y_stage_bytes = 0;
  size_t permute_end = 0, router_w3 = 0, router_end = 0;
  size_t sfa = 0, sfa_end = 0;  // MX plans: activation scale atoms of the permuted rows
};

}  // namespace

struct moe_plan_s {
  moe_layer_desc desc;
  moe_layer_weights w;
  int device;
  int ex, eh, ey;  // element bytes of x / hidden / y
  int dout;
  CUtensorMap tmW1, tmW3, tmW2;      // single-CTA tiles (256-row boxes; 128 for gate/up)
  CUtensorMap tmW1h, tmW2h;          // CTA-pair tiles: 128-row boxes
  Layout L;
  bool profile;
  cudaEvent_t ev[kMaxEvents];
  const char* ev_name[kMaxEvents];
  int nev;
  int launches;
  cudaStream_t h2d, d2h;  // host-buffer path copy streams (created on first use)
  cudaStream_t side;      // shared-expert stream of moe_forward_routed_shared (first use)
  cudaEvent_t sev[2];     // fork / join of that stream
  cudaEvent_t hev[kHostEvents];
  unsigned long long host_calls;  // host-buffer calls so far (selects the staging slot)
  uint8_t* sfb;  // MX plans: the weight scales in the tensor-core layout (owned)
  float* wgs;    // group / block plans: the weight scales, (E, d/128, F or F/128) (owned)
  void* router_w;  // the router weights split for the tensor-core routers (owned), or NULL
  int router_kind; // kRouterSimt, kRouterMma, kRouterTc
  CUtensorMap tmRouterW;  // kRouterTc: TMA map of the split router weights
};

namespace {

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device or managed memory (a kernel may read it); host or unknown pointers
// are refused before any launch.
bool device_accessible(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the error of an unregistered host pointer
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

// Stage boundary marker for the optional per-kernel timing.
void mark(moe_plan p, cudaStream_t s, const char* name_of_next) {
  if (!p->profile || p->nev >= kMaxEvents) return;
  cudaEventRecord(p->ev[p->nev], s);
  p->ev_name[p->nev] = name_of_next;
  p->nev++;
}

bool uses_tensor_cores(const moe_layer_desc& d) { return d.dtype != MOE_F32; }

enum RouterKind { kRouterSimt = 0, kRouterMma = 1, kRouterTc = 2 };

// Router flavour of a plan: split-K SIMT for few tokens with long rows;
// else, for bf16 tokens, the warp-MMA router (E <= 16) or the fused tcgen05
// router (33..128 experts), both on the plan's split copy of w_r, or the
// tcgen05 logits GEMM + top-K kernel on a per-call split in workspace
// scratch (more than 128 experts); else the per-token SIMT kernels.
bool router_splitk(const moe_layer_desc& d) { return router_uses_splitk(d.N, d.d); }
bool router_on_tensor_cores(const moe_layer_desc& d) {
  return !router_splitk(d) && d.dtype == MOE_BF16 && d.E > kRouterFusedMaxExperts;
}

void layout(moe_plan p) {
  const moe_layer_desc& d = p->desc;
  const long long R = static_cast<long long>(d.N) * d.K;
  Layout L;
  size_t off = 0;
  L.status = off; off = align_up(off + 4);
  L.counter = off; off = align_up(off + 4);  // the permute rank pass's last-CTA counter
  // the rank pass's per-block expert histograms, then block bases
  L.chunk_counts = off; off = align_up(off + permute_block_counts_bytes(d.N, d.E));
  L.permute_end = off;
  L.router_w3 = off;
  if (router_on_tensor_cores(d)) off = align_up(off + router_tc_scratch_bytes(d.N, d.d, d.E));
  if (router_splitk(d)) off = align_up(off + router_splitk_scratch_bytes(d.N, d.d, d.E));
  L.router_end = off;
  L.h = off;
  if (d.act != MOE_ACT_NONE) off = align_up(off + static_cast<size_t>(R) * d.F * p->eh);
  // fp32 layers: split-K partial sums of the SIMT GEMMs (up to 8 slices,
  // gate and up for SwiGLU), shared by the layer's GEMMs (they run in order)
  L.simt_part = off;
  if (!uses_tensor_cores(d))
    off = align_up(off + static_cast<size_t>(8) * 2 * R * (d.F > d.d ? d.F : d.d) * sizeof(float));
  L.h_end = off;
  L.ids = off; off = align_up(off + static_cast<size_t>(R) * 4);
  L.gates = off; off = align_up(off + static_cast<size_t>(R) * 4);
  L.pos = off; off = align_up(off + static_cast<size_t>(R) * 4);
  L.src = off; off = align_up(off + static_cast<size_t>(R) * 4);
  L.slot = off; off = align_up(off + static_cast<size_t>(R) * 4);
  L.tok_scale = off; off = align_up(off + static_cast<size_t>(d.N) * 4);
  L.counts = off; off = align_up(off + static_cast<size_t>(d.E) * 4);
  L.offsets = off; off = align_up(off + static_cast<size_t>(d.E + 1) * 4);
  L.x_perm = off; off = align_up(off + static_cast<size_t>(R) * d.d * p->ex);
  L.y_perm = off; off = align_up(off + static_cast<size_t>(R) * p->dout * p->ey);
  L.sfa = off;
  if (d.quant == MOE_QUANT_MX) off = align_up(off + mx_act_sf_bytes(R, d.E, d.d));
  L.sfa_end = off;
  L.fwd_end = off;
  // two staging slots for x and y: consecutive host-buffer calls alternate
  const size_t xbytes = align_up(static_cast<size_t>(d.N) * d.d * p->ex);
  const size_t ybytes = align_up(static_cast<size_t>(d.N) * p->dout * p->ey);
  L.x_stage = off; off += 2 * xbytes;
  L.y_stage = off; off += 2 * ybytes;
  L.x_stage_bytes = xbytes;
  L.y_stage_bytes = ybytes;
  L.total = off;
  p->L = L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

moe_status check_ws(moe_plan p, void* ws, size_t ws_bytes, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  (void)p;
  return MOE_OK;
}

// The stage runners take the token count n <= plan N explicitly (the
// host-buffer path runs the layer on token chunks).
moe_status run_router(moe_plan p, int n, const void* x, int32_t* ids, float* gates, float* margin,
                      void* ws, cudaStream_t s) {
  const moe_layer_desc& d = p->desc;
  if (p->router_kind == kRouterMma) {
    mark(p, s, "router_mma");
    p->launches += 1;
    return cuda_status(launch_router_mma(x, p->router_w, p->w.router_bias, n, d.d, d.E, d.K, ids,
                                         gates, margin, at<int>(ws, p->L.status), s));
  }
  if (p->router_kind == kRouterTc) {
    mark(p, s, "router_tc");
    p->launches += 1;  // logits and top-K in one kernel
    return cuda_status(launch_router_fused(x, p->tmRouterW, p->w.router_bias, n, d.d, d.E, d.K,
                                           ids, gates, margin, at<int>(ws, p->L.status), s));
  }
  if (router_on_tensor_cores(d)) {
    mark(p, s, "router_tc");
    p->launches += 3;  // weight split + logits + top-K
    return cuda_status(launch_router_tc(x, p->w.w_r, p->w.router_bias, n, d.d, d.E, d.K, ids, gates,
                                        margin, at<void>(ws, p->L.router_w3),
                                        at<int>(ws, p->L.status), s));
  }
  const bool splitk = router_splitk(d);
  mark(p, s, splitk ? "router_splitk" : "router_topk");
  p->launches += splitk ? 2 : 1;  // partial logits + reduction/top-K
  return cuda_status(launch_router(x, d.dtype, p->w.w_r, p->w.router_bias, n, d.d, d.E, d.K, ids,
                                   gates, margin, at<void>(ws, p->L.router_w3), s));
}

// slot (optional): slot[pos] = t*K + j, the destination row of a pure
// unpermute, for a grouped FFN that stores its rows there directly.
moe_status run_permute(moe_plan p, int n, const void* x, const int32_t* ids, int32_t* counts,
                       int32_t* offsets, int32_t* pos, int32_t* src, void* x_perm, void* ws,
                       cudaStream_t s, int32_t* slot = nullptr) {
  const moe_layer_desc& d = p->desc;
  int* status = at<int>(ws, p->L.status);
  int32_t* cc = at<int32_t>(ws, p->L.chunk_counts);
  // no rows to copy and a small batch: the rank pass also makes the positions
  const bool positions_in_rank =
      x_perm == nullptr && slot == nullptr &&
      static_cast<long long>(n) * d.K <= kRankPositionsMaxRows;
  mark(p, s, "permute_rank");
  if (launch_permute_rank(ids, n, d.K, d.E, cc, at<unsigned>(ws, p->L.counter), pos, counts,
                          offsets, status, s, positions_in_rank ? src : nullptr) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (positions_in_rank) {
    p->launches += 1;
    return MOE_OK;
  }
  mark(p, s, x_perm ? "permute_gather" : "permute_positions");
  if (launch_permute_gather(x, d.d * p->ex, ids, n, d.K, d.E, cc, pos, src, slot, x_perm, status,
                            s) != cudaSuccess)
    return MOE_ERR_CUDA;
  p->launches += 2;
  return MOE_OK;
}

// run_permute with per-token dynamic quantization of bf16 x into e4m3 x_perm.
moe_status run_permute_quant(moe_plan p, int n, const void* x_bf16, const int32_t* ids,
                             int32_t* counts, int32_t* offsets, int32_t* pos, int32_t* src,
                             void* x_perm, float* token_scales, void* ws, cudaStream_t s,
                             int32_t* slot = nullptr) {
  const moe_layer_desc& d = p->desc;
  int* status = at<int>(ws, p->L.status);
  int32_t* cc = at<int32_t>(ws, p->L.chunk_counts);
  mark(p, s, "permute_rank");
  if (launch_permute_rank(ids, n, d.K, d.E, cc, at<unsigned>(ws, p->L.counter), pos, counts,
                          offsets, status, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  mark(p, s, "permute_quant");
  if (launch_permute_quant(x_bf16, d.d, ids, n, d.K, d.E, cc, pos, src, slot, x_perm,
                           token_scales, status, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  p->launches += 2;
  return MOE_OK;
}

// Whether the whole-layer call of a bf16 SwiGLU plan gathers the gate/up
// GEMM's A rows straight from the tokens (no row copy in the permute): for
// decode-shaped batches, at most kGatherRowsPerExpert routed rows per expert
// on average, where each stage's A tile is a few rows beside 256 weight rows
// (for larger batches a 128-row A box per stage, copied once by the permute,
// is cheaper than re-gathering it for every column tile).
constexpr int kGatherRowsPerExpert = 16;
bool gather_fused(const moe_layer_desc& d, int n) {
  return d.dtype == MOE_BF16 && d.act == MOE_ACT_SWIGLU &&
         static_cast<long long>(n) * d.K <= static_cast<long long>(kGatherRowsPerExpert) * d.E;
}

// x_rows: per-token activation scales indexed by row_index[row] (or by the
// permuted row itself when row_index is NULL); NULL = the scalar x_scale.
// out_rows (tensor cores, single-matrix layer): result row r goes to row
// out_rows[r] of y_perm (the pure unpermute done by the GEMM's stores).
// x_tokens, a_rows (bf16 SwiGLU): the gate/up GEMM takes its A rows from the
// token rows, row r = x_tokens[a_rows[r]], instead of x_perm.
moe_status run_ffn(moe_plan p, int n, const void* x_perm, const int32_t* offsets, float x_scale,
                   const float* x_rows, const int32_t* row_index, void* y_perm, void* ws,
                   cudaStream_t s, const int32_t* out_rows = nullptr,
                   const void* x_tokens = nullptr, const int32_t* a_rows = nullptr) {
  const moe_layer_desc& d = p->desc;
  if (d.quant == MOE_QUANT_MX || d.quant == MOE_QUANT_PER_GROUP || d.quant == MOE_QUANT_PER_BLOCK)
    return MOE_ERR_UNSUPPORTED;  // the _mx / _group_scales calls carry the scales
  const int R = n * d.K;
  int* status = at<int>(ws, p->L.status);
  void* h = at<void>(ws, p->L.h);
  if (!uses_tensor_cores(d)) {
    const float* A = static_cast<const float*>(x_perm);
    float* part = at<float>(ws, p->L.simt_part);
    auto launches = [&](int kdim, int ncols) { return simt_f32_splits(kdim, ncols, R, d.E) > 1 ? 2 : 1; };
    if (d.act == MOE_ACT_NONE) {
      mark(p, s, "ffn_simt_f32");
      p->launches += launches(d.d, d.F);
      return cuda_status(launch_gemm_simt_f32(A, d.d, static_cast<const float*>(p->w.w1), nullptr,
                                              d.F, kActNone, 1.f, offsets, d.E, R,
                                              static_cast<float*>(y_perm), part, s));
    }
    mark(p, s, "ffn1_simt_f32");
    if (launch_gemm_simt_f32(A, d.d, static_cast<const float*>(p->w.w1),
                             static_cast<const float*>(p->w.w3), d.F, d.act, 1.f, offsets, d.E, R,
                             static_cast<float*>(h), part, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    mark(p, s, "ffn2_simt_f32");
    p->launches += launches(d.d, d.F) + launches(d.F, d.d);
    return cuda_status(launch_gemm_simt_f32(static_cast<const float*>(h), d.F,
                                            static_cast<const float*>(p->w.w2), nullptr, d.d,
                                            kActNone, 1.f, offsets, d.E, R,
                                            static_cast<float*>(y_perm), part, s));
  }
  TcGemmArgs a;
  memset(&a, 0, sizeof(a));
  a.offsets = offsets;
  a.groups = d.E;
  a.m_total = R;
  a.status = status;
  // 256-row tiles on CTA pairs when the experts average at least 512 routed
  // rows; below that the last, partly empty row tile of each expert wastes
  // too much MMA work and 128-row tiles on single CTAs win.  The SwiGLU
  // gate/up GEMM (short k loop, 128 outputs per tile) only pairs from 2048
  // rows per expert: at ~1024 its single-CTA tiles were 3 % faster, while
  // the down GEMM was 6-9 % faster paired (measured on one B200).
  const bool pair = R >= 512 * d.E;
  const bool pair_swiglu = R >= 2048 * d.E;
  // with no rows the GEMM schedules no tile; a map of one row keeps it valid
  const int map_rows = R > 0 ? R : 1;
  if (!encode_kmajor_map(&a.tmA, x_perm, p->ex, map_rows, d.d, kTcBlockM)) return MOE_ERR_CUDA;
  if (d.act == MOE_ACT_NONE) {
    a.tmB0 = pair ? p->tmW1h : p->tmW1;
    a.tmB1 = a.tmB0;
    a.kdim = d.d;
    a.n_out = d.F;
    a.n_tiles = (d.F + kTcBlockN - 1) / kTcBlockN;
    a.out = y_perm;
    a.out_rows = out_rows;
    a.ldo = d.F;
    if (d.dtype == MOE_E4M3) {
      const bool per_channel = d.quant == MOE_QUANT_PER_CHANNEL;
      a.scale = (x_rows ? 1.f : x_scale) * (per_channel ? 1.f : p->w.w_scale);
      a.row_scale = x_rows;
      a.row_index = x_rows ? row_index : nullptr;
      a.col_scale = per_channel ? p->w.w_channel_scales : nullptr;
    } else {
      a.scale = 1.f;
    }
    mark(p, s, "gmm_tc");
    p->launches += 1;
    return cuda_status(launch_gemm_tc(a, d.dtype, kEpiStore, R, pair, s));
  }
  // SwiGLU: gate/up GEMM with the activation fused into its epilogue, then down
  if (x_tokens != nullptr && a_rows != nullptr && !pair_swiglu) {
    if (!encode_kmajor_map(&a.tmAg, x_tokens, p->ex, n > 0 ? n : 1, d.d, 1)) return MOE_ERR_CUDA;
    a.a_rows = a_rows;
  }
  a.tmB0 = p->tmW1;
  a.tmB1 = p->tmW3;
  a.kdim = d.d;
  a.n_out = d.F;
  a.n_tiles = (d.F + kTcBlockN / 2 - 1) / (kTcBlockN / 2);
  a.out = h;
  a.ldo = d.F;
  a.out_tma = R > 0 && encode_out_map(&a.tmOut, h, R, d.F, d.F) ? 1 : 0;
  a.scale = 1.f;
  mark(p, s, a.a_rows ? "ffn1_swiglu_tc_gather" : "ffn1_swiglu_tc");
  if (launch_gemm_tc(a, d.dtype, kEpiSwiglu, R, pair_swiglu, s) != cudaSuccess) return MOE_ERR_CUDA;
  TcGemmArgs b = a;
  b.a_rows = nullptr;
  if (!encode_kmajor_map(&b.tmA, h, p->eh, map_rows, d.F, kTcBlockM)) return MOE_ERR_CUDA;
  b.tmB0 = pair ? p->tmW2h : p->tmW2;
  b.tmB1 = b.tmB0;
  b.kdim = d.F;
  b.n_out = d.d;
  b.n_tiles = (d.d + kTcBlockN - 1) / kTcBlockN;
  b.out = y_perm;
  b.ldo = d.d;
  b.out_tma = R > 0 && encode_out_map(&b.tmOut, y_perm, R, d.d, d.d) ? 1 : 0;
  mark(p, s, "ffn2_tc");
  p->launches += 2;
  return cuda_status(launch_gemm_tc(b, d.dtype, kEpiStore, R, pair, s));
}

// MX grouped matmul: the activation scales of the permuted rows are already
// in ws at L.sfa (tensor-core layout); out_rows as run_ffn.
moe_status run_ffn_mx(moe_plan p, int n, const void* x_perm, const int32_t* offsets, void* y_perm,
                      void* ws, cudaStream_t s, const int32_t* out_rows = nullptr) {
  const moe_layer_desc& d = p->desc;
  const int R = n * d.K;
  TcGemmArgs a;
  memset(&a, 0, sizeof(a));
  if (!encode_kmajor_map(&a.tmA, x_perm, 1, R > 0 ? R : 1, d.d, kTcBlockM)) return MOE_ERR_CUDA;
  a.tmB0 = p->tmW1;
  a.tmB1 = a.tmB0;
  a.offsets = offsets;
  a.groups = d.E;
  a.m_total = R;
  a.kdim = d.d;
  a.n_out = d.F;
  a.n_tiles = (d.F + kTcBlockN - 1) / kTcBlockN;
  a.out = y_perm;
  a.out_rows = out_rows;
  a.ldo = d.F;
  a.scale = 1.f;
  a.status = at<int>(ws, p->L.status);
  a.sfa = at<uint8_t>(ws, p->L.sfa);
  a.sfb = p->sfb;
  mark(p, s, "gmm_mx_tc");
  p->launches += 1;
  return cuda_status(launch_gemm_tc(a, kGemmMxE4M3, kEpiStore, R, false, s));
}

// Group / block-scaled grouped matmul (quant modes 4, 5).  Activation
// scales: x_group (per row and 128-element group, indexed through
// row_index), else x_rows (per row), else x_scale.
moe_status run_ffn_gs(moe_plan p, int n, const void* x_perm, const int32_t* offsets, float x_scale,
                      const float* x_rows, const float* x_group, const int32_t* row_index,
                      void* y_perm, void* ws, cudaStream_t s, const int32_t* out_rows = nullptr) {
  const moe_layer_desc& d = p->desc;
  const int R = n * d.K;
  TcGemmArgs a;
  memset(&a, 0, sizeof(a));
  if (!encode_kmajor_map(&a.tmA, x_perm, 1, R > 0 ? R : 1, d.d, kTcBlockM)) return MOE_ERR_CUDA;
  const bool blocks = d.quant == MOE_QUANT_PER_BLOCK;
  // per-column scales: 128 x 128 tiles (128-row weight boxes); block scales:
  // 128 x 256 tiles
  a.tmB0 = blocks ? p->tmW1 : p->tmW1h;
  a.tmB1 = a.tmB0;
  a.offsets = offsets;
  a.groups = d.E;
  a.m_total = R;
  a.kdim = d.d;
  a.n_out = d.F;
  const int tile_n = blocks ? kTcBlockN : kGsTileN;
  a.n_tiles = (d.F + tile_n - 1) / tile_n;
  a.out = y_perm;
  a.out_rows = out_rows;
  a.ldo = d.F;
  a.scale = x_group || x_rows ? 1.f : x_scale;
  a.row_scale = x_group ? nullptr : x_rows;
  a.row_index = row_index;
  a.xgs = x_group;
  a.wgs = p->wgs;
  a.status = at<int>(ws, p->L.status);
  mark(p, s, blocks ? "gmm_block_tc" : "gmm_group_tc");
  p->launches += 1;
  return cuda_status(blocks ? launch_gemm_tc(a, kE4M3, kEpiBlockScale, R, false, s)
                            : launch_gemm_gs(a, R, s));
}

moe_status run_combine(moe_plan p, int n, const void* y_perm, const int32_t* pos,
                       const float* gates, void* y, void* ws, cudaStream_t s) {
  const moe_layer_desc& d = p->desc;
  mark(p, s, gates ? "combine" : "unpermute");
  p->launches += 1;
  const int ydt = d.dtype == MOE_F32 ? kF32 : kBF16;
  return cuda_status(launch_combine(y_perm, ydt, p->dout, pos, gates, n, d.K, y,
                                    at<int>(ws, p->L.status), s));
}

void begin(moe_plan p) {
  p->nev = 0;
  p->launches = 0;
}
void end(moe_plan p, cudaStream_t s) { mark(p, s, nullptr); }

}  // namespace

extern "C" {

const char* moe_status_string(moe_status st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_BAD_INDEX: return "device: index out of range";
    case MOE_ERR_DEVICE_TIMEOUT: return "device: pipeline wait timed out";
  }
  return "unknown status";
}

moe_status moe_plan_create(const moe_layer_desc* desc, const moe_layer_weights* w, moe_plan* out) {
  if (!desc || !w || !out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const moe_layer_desc d = *desc;
  // limits of the Ascend page (K in [2, 8] widened to [1, 8]; experts <= 256;
  // H1, N1 < 65536)
  if (d.N < 1 || d.d < 1 || d.d >= 65536 || d.E < 1 || d.E > 256 || d.K < 1 || d.K > 8 ||
      d.K > d.E || d.F < 1 || d.F >= 65536)
    return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(d.N) * d.K >= (1LL << 31)) return MOE_ERR_INVALID_ARG;
  if (d.dtype < MOE_F32 || d.dtype > MOE_E4M3 || d.act < MOE_ACT_NONE || d.act > MOE_ACT_SWIGLU ||
      d.quant < MOE_QUANT_NONE || d.quant > MOE_QUANT_MX)
    return MOE_ERR_INVALID_ARG;
  // modes 3 (per-token) and 7 (dynamic) are per-call arguments
  if (d.quant == 3) return MOE_ERR_UNSUPPORTED;
  const bool gs = d.quant == MOE_QUANT_PER_GROUP || d.quant == MOE_QUANT_PER_BLOCK;
  if ((d.quant != MOE_QUANT_NONE) != (d.dtype == MOE_E4M3)) return MOE_ERR_UNSUPPORTED;
  if ((d.quant == MOE_QUANT_PER_CHANNEL) != (w->w_channel_scales != nullptr))
    return MOE_ERR_INVALID_ARG;
  if (d.quant != MOE_QUANT_MX && w->w_mx_scales) return MOE_ERR_INVALID_ARG;
  if (!gs && w->w_group_scales) return MOE_ERR_INVALID_ARG;
  if (gs && (d.d % 128 || (w->w1 && !w->w_group_scales))) return MOE_ERR_INVALID_ARG;
  if (d.quant == MOE_QUANT_MX && (d.d % kMxBlock || d.d > kMxMaxKdim || (w->w1 && !w->w_mx_scales)))
    return MOE_ERR_INVALID_ARG;
  if (d.dtype == MOE_E4M3 && d.act != MOE_ACT_NONE) return MOE_ERR_UNSUPPORTED;
  if (d.dtype == MOE_BF16 && d.act == MOE_ACT_RELU) return MOE_ERR_UNSUPPORTED;
  // a routing-only plan (no expert weights: router, permute and combine of
  // an expert-parallel layer whose experts live on other GPUs) takes none of
  // w1, w3, w2
  const bool routing_only = !w->w1 && !w->w3 && !w->w2 && d.quant != MOE_QUANT_PER_CHANNEL &&
                            !w->w_mx_scales && !w->w_group_scales;
  if (!routing_only && (!w->w1 || (d.act == MOE_ACT_SWIGLU) != (w->w3 != nullptr) ||
                        (d.act != MOE_ACT_NONE) != (w->w2 != nullptr)))
    return MOE_ERR_INVALID_ARG;
  if ((w->w1 && !aligned16(w->w1)) || (w->w3 && !aligned16(w->w3)) || (w->w2 && !aligned16(w->w2)) ||
      (w->w_r && !aligned16(w->w_r)))
    return MOE_ERR_INVALID_ARG;

  moe_plan p = new (std::nothrow) moe_plan_s;
  if (!p) return MOE_ERR_CUDA;
  memset(static_cast<void*>(p), 0, sizeof(*p));
  p->desc = d;
  p->w = *w;
  p->ex = dtype_bytes(d.dtype);
  p->eh = d.dtype == MOE_F32 ? 4 : 2;
  p->ey = d.dtype == MOE_F32 ? 4 : 2;
  p->dout = d.act == MOE_ACT_NONE ? d.F : d.d;
  // every row that a kernel moves with 16-byte vectors or TMA is a multiple
  // of 16 bytes
  if ((static_cast<long long>(d.d) * p->ex) % 16 || (static_cast<long long>(p->dout) * p->ey) % 16 ||
      (d.act != MOE_ACT_NONE && (static_cast<long long>(d.F) * p->eh) % 16)) {
    delete p;
    return MOE_ERR_INVALID_ARG;
  }
  if (cudaGetDevice(&p->device) != cudaSuccess) {
    delete p;
    return MOE_ERR_CUDA;
  }
  if (uses_tensor_cores(d) && !routing_only) {
    bool ok = true;
    const long long rows1 = static_cast<long long>(d.E) * d.F;
    if (d.act == MOE_ACT_NONE) {
      ok = encode_kmajor_map(&p->tmW1, w->w1, p->ex, rows1, d.d, kTcBlockN) &&
           encode_kmajor_map(&p->tmW1h, w->w1, p->ex, rows1, d.d, kTcBlockN / 2);
    } else {
      const long long rows2 = static_cast<long long>(d.E) * d.d;
      ok = encode_kmajor_map(&p->tmW1, w->w1, p->ex, rows1, d.d, kTcBlockN / 2) &&
           encode_kmajor_map(&p->tmW3, w->w3, p->ex, rows1, d.d, kTcBlockN / 2) &&
           encode_kmajor_map(&p->tmW2, w->w2, p->ex, rows2, d.F, kTcBlockN) &&
           encode_kmajor_map(&p->tmW2h, w->w2, p->ex, rows2, d.F, kTcBlockN / 2);
    }
    if (!ok) {
      delete p;
      return MOE_ERR_CUDA;
    }
  }
  // the plan-time kernels below read the scale tables: refuse host pointers
  if ((d.quant == MOE_QUANT_MX && !routing_only && !device_accessible(w->w_mx_scales)) ||
      (gs && !routing_only && !device_accessible(w->w_group_scales))) {
    delete p;
    return MOE_ERR_INVALID_ARG;
  }
  if (d.quant == MOE_QUANT_MX && !routing_only) {
    // the weight scales, once, in the layout the block-scaled GEMM reads
    cudaStream_t cs = nullptr;
    const size_t bytes = mx_weight_sf_bytes(d.E, d.F, d.d);
    bool ok = cudaMalloc(reinterpret_cast<void**>(&p->sfb), bytes) == cudaSuccess;
    ok = ok && cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) == cudaSuccess;
    ok = ok && launch_mx_weight_sf(w->w_mx_scales, d.E, d.F, d.d, p->sfb, cs) == cudaSuccess;
    ok = ok && cudaStreamSynchronize(cs) == cudaSuccess;
    if (cs) cudaStreamDestroy(cs);
    if (!ok) {
      if (p->sfb) cudaFree(p->sfb);
      delete p;
      return MOE_ERR_CUDA;
    }
  }
  if (gs && !routing_only) {
    // the weight scales, once, transposed to (E, d/128, columns): a stage's
    // scales are contiguous for the epilogue (256 floats of slack at the end
    // for its vector loads past the last column)
    const int ng = d.d / 128;
    const int cols = d.quant == MOE_QUANT_PER_BLOCK ? (d.F + 127) / 128 : d.F;
    const size_t bytes = (static_cast<size_t>(d.E) * ng * cols + 256) * sizeof(float);
    cudaStream_t cs = nullptr;
    bool ok = cudaMalloc(reinterpret_cast<void**>(&p->wgs), bytes) == cudaSuccess;
    ok = ok && cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) == cudaSuccess;
    ok = ok && cudaMemsetAsync(p->wgs, 0, bytes, cs) == cudaSuccess;
    ok = ok && launch_group_scales_t(w->w_group_scales, d.E, cols, ng, p->wgs, cs) == cudaSuccess;
    ok = ok && cudaStreamSynchronize(cs) == cudaSuccess;
    if (cs) cudaStreamDestroy(cs);
    if (!ok) {
      if (p->wgs) cudaFree(p->wgs);
      delete p;
      return MOE_ERR_CUDA;
    }
  }
  for (int i = 0; i < kMaxEvents; ++i) p->ev[i] = nullptr;
  layout(p);
  // the router weights, once, in the layout of the plan's tensor-core router
  p->router_kind = kRouterSimt;
  if (w->w_r && router_uses_mma(d.N, d.d, d.E, d.dtype)) p->router_kind = kRouterMma;
  if (w->w_r && router_uses_fused_tc(d.N, d.d, d.E, d.dtype)) p->router_kind = kRouterTc;
  if (p->router_kind != kRouterSimt) {
    if (!device_accessible(w->w_r)) {
      moe_plan_destroy(p);
      return MOE_ERR_INVALID_ARG;
    }
    const size_t bytes = p->router_kind == kRouterMma ? router_mma_frag_bytes(d.d, d.E)
                                                      : router_fused_weight_bytes(d.d, d.E);
    cudaStream_t cs = nullptr;
    bool ok = cudaMalloc(&p->router_w, bytes) == cudaSuccess;
    ok = ok && (p->router_kind != kRouterTc ||
                encode_router_fused_weights(&p->tmRouterW, p->router_w, d.d, d.E));
    ok = ok && cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) == cudaSuccess;
    ok = ok && moe_plan_refresh_router(p, cs) == MOE_OK;
    ok = ok && cudaStreamSynchronize(cs) == cudaSuccess;
    if (cs) cudaStreamDestroy(cs);
    if (!ok) {
      moe_plan_destroy(p);
      return MOE_ERR_CUDA;
    }
  }
  *out = p;
  return MOE_OK;
}

moe_status moe_plan_refresh_router(moe_plan p, moe_stream_t stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (p->router_kind == kRouterSimt || !p->w.w_r) return MOE_OK;  // reads w_r on every call
  const moe_layer_desc& d = p->desc;
  if (p->router_kind == kRouterMma)
    return cuda_status(launch_router_mma_frag(p->w.w_r, d.d, d.E, p->router_w, stream));
  return cuda_status(launch_router_fused_split(p->w.w_r, d.d, d.E, p->router_w, stream));
}

moe_status moe_plan_destroy(moe_plan p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < kMaxEvents; ++i)
    if (p->ev[i]) cudaEventDestroy(p->ev[i]);
  for (int i = 0; i < kHostEvents; ++i)
    if (p->hev[i]) cudaEventDestroy(p->hev[i]);
  if (p->h2d) cudaStreamDestroy(p->h2d);
  if (p->d2h) cudaStreamDestroy(p->d2h);
  for (int i = 0; i < 2; ++i)
    if (p->sev[i]) cudaEventDestroy(p->sev[i]);
  if (p->side) cudaStreamDestroy(p->side);
  if (p->sfb) cudaFree(p->sfb);
  if (p->wgs) cudaFree(p->wgs);
  if (p->router_w) cudaFree(p->router_w);
  delete p;
  return MOE_OK;
}

moe_status moe_workspace_size(moe_plan p, size_t* bytes) {
  if (!p || !bytes) return MOE_ERR_INVALID_ARG;
  *bytes = p->L.total;
  return MOE_OK;
}

moe_status moe_workspace_init(moe_plan p, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.chunk_counts);
  if (st != MOE_OK) return st;
  // the status word and the permute's counter
  return cuda_status(cudaMemsetAsync(ws, 0, p->L.chunk_counts, stream));
}

moe_status moe_router_topk(moe_plan p, const void* x, int32_t* ids, float* gates, float* margin,
                           void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x || !ids || !gates || !p->w.w_r) return MOE_ERR_INVALID_ARG;
  if (p->desc.dtype == MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
  moe_status st0 = check_ws(p, ws, ws_bytes, p->L.router_end);
  if (st0 != MOE_OK) return st0;
  begin(p);
  moe_status st = run_router(p, p->desc.N, x, ids, gates, margin, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_permute_n(moe_plan p, int32_t n, const void* x, const int32_t* ids,
                         int32_t* counts, int32_t* offsets, int32_t* pos, int32_t* src,
                         void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x || !ids || !counts || !offsets || !pos || !src || !x_perm) return MOE_ERR_INVALID_ARG;
  if (n < 0 || n > p->desc.N) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.permute_end);
  if (st != MOE_OK) return st;
  begin(p);
  st = run_permute(p, n, x, ids, counts, offsets, pos, src, x_perm, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_permute(moe_plan p, const void* x, const int32_t* ids, int32_t* counts,
                       int32_t* offsets, int32_t* pos, int32_t* src, void* x_perm, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  return moe_permute_n(p, p->desc.N, x, ids, counts, offsets, pos, src, x_perm, ws, ws_bytes,
                       stream);
}

moe_status moe_grouped_ffn_n(moe_plan p, int32_t n, const void* x_perm, const int32_t* offsets,
                             float x_scale, const float* x_row_scales, void* y_perm, void* ws,
                             size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x_perm || !offsets || !y_perm) return MOE_ERR_INVALID_ARG;
  if (n < 0 || n > p->desc.N) return MOE_ERR_INVALID_ARG;
  if (!p->w.w1) return MOE_ERR_UNSUPPORTED;  // routing-only plan
  if (!aligned16(x_perm) || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.h_end);
  if (st != MOE_OK) return st;
  begin(p);
  st = run_ffn(p, n, x_perm, offsets, x_scale, x_row_scales, nullptr, y_perm, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_grouped_ffn(moe_plan p, const void* x_perm, const int32_t* offsets, float x_scale,
                           const float* x_row_scales, void* y_perm, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  return moe_grouped_ffn_n(p, p->desc.N, x_perm, offsets, x_scale, x_row_scales, y_perm, ws,
                           ws_bytes, stream);
}

moe_status moe_unpermute_combine_n(moe_plan p, int32_t n, const void* y_perm,
                                   const int32_t* pos, const float* gates, void* y, void* ws,
                                   size_t ws_bytes, moe_stream_t stream) {
  if (!p || !y_perm || !pos || !y) return MOE_ERR_INVALID_ARG;
  if (n < 0 || n > p->desc.N) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.chunk_counts);
  if (st != MOE_OK) return st;
  begin(p);
  st = run_combine(p, n, y_perm, pos, gates, y, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_unpermute_combine(moe_plan p, const void* y_perm, const int32_t* pos,
                                 const float* gates, void* y, void* ws, size_t ws_bytes,
                                 moe_stream_t stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  return moe_unpermute_combine_n(p, p->desc.N, y_perm, pos, gates, y, ws, ws_bytes, stream);
}

moe_status moe_shared_matmul(moe_plan p, const void* x, int32_t M, int32_t H, const void* w,
                             int32_t N2, float x_scale, const float* x_token_scales,
                             float w_scale, const float* w_channel_scales, void* y,
                             moe_stream_t stream) {
  if (!p || !x || !w || !y || M < 1 || H < 16 || H > 12288 || H % 16 || N2 < 1 || N2 >= 65536 ||
      N2 % 8)
    return MOE_ERR_INVALID_ARG;
  if (p->desc.dtype != MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  TcGemmArgs a;
  memset(&a, 0, sizeof(a));
  const bool pair = M >= 256;
  if (!encode_kmajor_map(&a.tmA, x, 1, M, H, kTcBlockM) ||
      !encode_kmajor_map(&a.tmB0, w, 1, N2, H, pair ? kTcBlockN / 2 : kTcBlockN))
    return MOE_ERR_CUDA;
  a.tmB1 = a.tmB0;
  a.offsets = nullptr;
  a.groups = 1;
  a.m_total = M;
  a.kdim = H;
  a.n_out = N2;
  a.n_tiles = (N2 + kTcBlockN - 1) / kTcBlockN;
  a.out = y;
  a.ldo = N2;
  a.scale = (x_token_scales ? 1.f : x_scale) * (w_channel_scales ? 1.f : w_scale);
  a.row_scale = x_token_scales;
  a.col_scale = w_channel_scales;
  a.status = nullptr;
  return cuda_status(launch_gemm_tc(a, kE4M3, kEpiStore, M, pair, stream));
}

moe_status moe_forward_routed(moe_plan p, const void* x, const int32_t* ids, const float* gates,
                              float x_scale, const float* x_token_scales, void* y, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x || !ids || !y) return MOE_ERR_INVALID_ARG;
  if (!p->w.w1) return MOE_ERR_UNSUPPORTED;  // routing-only plan
  if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.fwd_end);
  if (st != MOE_OK) return st;
  const Layout& L = p->L;
  begin(p);
  const int n = p->desc.N;
  int32_t* src = at<int32_t>(ws, L.src);
  // a pure unpermute of the single-matrix layer on the tensor cores is done
  // by the GEMM's stores (row r -> row slot[r] = t*K + j of y): no reorder pass
  const bool scatter = uses_tensor_cores(p->desc) && p->desc.act == MOE_ACT_NONE && !gates;
  int32_t* slot = scatter ? at<int32_t>(ws, L.slot) : nullptr;
  st = run_permute(p, n, x, ids, at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets),
                   at<int32_t>(ws, L.pos), src, at<void>(ws, L.x_perm), ws, stream, slot);
  // per-token scales reach the permuted rows through the source-token index
  if (st == MOE_OK)
    st = run_ffn(p, n, at<void>(ws, L.x_perm), at<int32_t>(ws, L.offsets), x_scale,
                 x_token_scales, src, scatter ? y : at<void>(ws, L.y_perm), ws, stream, slot);
  if (st == MOE_OK && !scatter)
    st = run_combine(p, n, at<void>(ws, L.y_perm), at<int32_t>(ws, L.pos), gates, y, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_permute_mx(moe_plan p, const void* x, const uint8_t* x_mx_scales,
                          const int32_t* ids, int32_t* counts, int32_t* offsets, int32_t* pos,
                          int32_t* src, void* x_perm, uint8_t* x_perm_mx_scales, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x || !x_mx_scales || !ids || !counts || !offsets || !pos || !src || !x_perm ||
      !x_perm_mx_scales)
    return MOE_ERR_INVALID_ARG;
  if (p->desc.quant != MOE_QUANT_MX) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.permute_end);
  if (st != MOE_OK) return st;
  const moe_layer_desc& d = p->desc;
  begin(p);
  st = run_permute(p, d.N, x, ids, counts, offsets, pos, src, x_perm, ws, stream);
  if (st == MOE_OK) {
    mark(p, stream, "mx_sf_gather");
    p->launches += 1;
    st = cuda_status(launch_mx_sf_gather(x_mx_scales, src, offsets, d.E, d.N * d.K,
                                         d.d / kMxBlock, x_perm_mx_scales, stream));
  }
  end(p, stream);
  return st;
}

moe_status moe_grouped_ffn_mx(moe_plan p, const void* x_perm, const uint8_t* x_perm_mx_scales,
                              const int32_t* offsets, void* y_perm, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  if (!p || !x_perm || !x_perm_mx_scales || !offsets || !y_perm) return MOE_ERR_INVALID_ARG;
  if (p->desc.quant != MOE_QUANT_MX) return MOE_ERR_UNSUPPORTED;
  if (!p->w.w1) return MOE_ERR_UNSUPPORTED;  // routing-only plan
  if (!aligned16(x_perm) || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.sfa_end);
  if (st != MOE_OK) return st;
  const moe_layer_desc& d = p->desc;
  const int R = d.N * d.K;
  begin(p);
  mark(p, stream, "mx_act_sf");
  p->launches += 1;
  st = cuda_status(launch_mx_act_sf(x_perm_mx_scales, nullptr, offsets, d.E, R, d.d,
                                    at<uint8_t>(ws, p->L.sfa), stream));
  if (st == MOE_OK) st = run_ffn_mx(p, d.N, x_perm, offsets, y_perm, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_forward_routed_mx(moe_plan p, const void* x, const uint8_t* x_mx_scales,
                                 const int32_t* ids, const float* gates, void* y, void* ws,
                                 size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x || !x_mx_scales || !ids || !y) return MOE_ERR_INVALID_ARG;
  if (p->desc.quant != MOE_QUANT_MX) return MOE_ERR_UNSUPPORTED;
  if (!p->w.w1) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.fwd_end);
  if (st != MOE_OK) return st;
  const moe_layer_desc& d = p->desc;
  const Layout& L = p->L;
  begin(p);
  int32_t* src = at<int32_t>(ws, L.src);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* slot = gates ? nullptr : at<int32_t>(ws, L.slot);  // unpermute by the GEMM's stores
  st = run_permute(p, d.N, x, ids, at<int32_t>(ws, L.counts), offsets, at<int32_t>(ws, L.pos), src,
                   at<void>(ws, L.x_perm), ws, stream, slot);
  if (st == MOE_OK) {
    // each permuted row's scales come from its source token's row
    mark(p, stream, "mx_act_sf");
    p->launches += 1;
    st = cuda_status(launch_mx_act_sf(x_mx_scales, src, offsets, d.E, d.N * d.K, d.d,
                                      at<uint8_t>(ws, L.sfa), stream));
  }
  if (st == MOE_OK)
    st = run_ffn_mx(p, d.N, at<void>(ws, L.x_perm), offsets, gates ? at<void>(ws, L.y_perm) : y, ws,
                    stream, slot);
  if (st == MOE_OK && gates)
    st = run_combine(p, d.N, at<void>(ws, L.y_perm), at<int32_t>(ws, L.pos), gates, y, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_grouped_ffn_group_scales(moe_plan p, const void* x_perm, float x_scale,
                                        const float* x_row_scales, const float* x_group_scales,
                                        const int32_t* offsets, void* y_perm, void* ws,
                                        size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x_perm || !offsets || !y_perm) return MOE_ERR_INVALID_ARG;
  if (p->desc.quant != MOE_QUANT_PER_GROUP && p->desc.quant != MOE_QUANT_PER_BLOCK)
    return MOE_ERR_UNSUPPORTED;
  if (!p->w.w1) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x_perm) || !aligned16(y_perm)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.permute_end);
  if (st != MOE_OK) return st;
  begin(p);
  st = run_ffn_gs(p, p->desc.N, x_perm, offsets, x_scale, x_row_scales, x_group_scales, nullptr,
                  y_perm, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_forward_routed_group_scales(moe_plan p, const void* x, float x_scale,
                                           const float* x_token_scales,
                                           const float* x_group_scales, const int32_t* ids,
                                           const float* gates, void* y, void* ws,
                                           size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x || !ids || !y) return MOE_ERR_INVALID_ARG;
  if (p->desc.quant != MOE_QUANT_PER_GROUP && p->desc.quant != MOE_QUANT_PER_BLOCK)
    return MOE_ERR_UNSUPPORTED;
  if (!p->w.w1) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.fwd_end);
  if (st != MOE_OK) return st;
  const moe_layer_desc& d = p->desc;
  const Layout& L = p->L;
  begin(p);
  int32_t* src = at<int32_t>(ws, L.src);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* slot = gates ? nullptr : at<int32_t>(ws, L.slot);  // unpermute by the GEMM's stores
  st = run_permute(p, d.N, x, ids, at<int32_t>(ws, L.counts), offsets, at<int32_t>(ws, L.pos), src,
                   at<void>(ws, L.x_perm), ws, stream, slot);
  // the activation scales reach the permuted rows through the source token
  if (st == MOE_OK)
    st = run_ffn_gs(p, d.N, at<void>(ws, L.x_perm), offsets, x_scale, x_token_scales,
                    x_group_scales, src, gates ? at<void>(ws, L.y_perm) : y, ws, stream, slot);
  if (st == MOE_OK && gates)
    st = run_combine(p, d.N, at<void>(ws, L.y_perm), at<int32_t>(ws, L.pos), gates, y, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_permute_quant(moe_plan p, const void* x_bf16, const int32_t* ids, int32_t* counts,
                             int32_t* offsets, int32_t* pos, int32_t* src, void* x_perm,
                             float* token_scales, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x_bf16 || !ids || !counts || !offsets || !pos || !src || !x_perm || !token_scales)
    return MOE_ERR_INVALID_ARG;
  if (p->desc.dtype != MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x_bf16) || !aligned16(x_perm) || p->desc.d % 16) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.permute_end);
  if (st != MOE_OK) return st;
  begin(p);
  st = run_permute_quant(p, p->desc.N, x_bf16, ids, counts, offsets, pos, src, x_perm,
                         token_scales, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_forward_routed_dynamic(moe_plan p, const void* x_bf16, const int32_t* ids,
                                      const float* gates, void* y, void* ws, size_t ws_bytes,
                                      moe_stream_t stream) {
  if (!p || !x_bf16 || !ids || !y) return MOE_ERR_INVALID_ARG;
  if (p->desc.dtype != MOE_E4M3 || !p->w.w1) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x_bf16) || !aligned16(y) || p->desc.d % 16) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.fwd_end);
  if (st != MOE_OK) return st;
  const Layout& L = p->L;
  begin(p);
  const int n = p->desc.N;
  int32_t* src = at<int32_t>(ws, L.src);
  float* tok = at<float>(ws, L.tok_scale);
  const bool scatter = p->desc.act == MOE_ACT_NONE && !gates;
  int32_t* slot = scatter ? at<int32_t>(ws, L.slot) : nullptr;
  st = run_permute_quant(p, n, x_bf16, ids, at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets),
                         at<int32_t>(ws, L.pos), src, at<void>(ws, L.x_perm), tok, ws, stream,
                         slot);
  // each permuted row takes its token's scale through the source-token index
  if (st == MOE_OK)
    st = run_ffn(p, n, at<void>(ws, L.x_perm), at<int32_t>(ws, L.offsets), 1.f, tok, src,
                 scatter ? y : at<void>(ws, L.y_perm), ws, stream, slot);
  if (st == MOE_OK && !scatter)
    st = run_combine(p, n, at<void>(ws, L.y_perm), at<int32_t>(ws, L.pos), gates, y, ws, stream);
  end(p, stream);
  return st;
}

moe_status moe_forward_routed_shared(moe_plan p, const void* x, const int32_t* ids,
                                     const float* gates, float x_scale,
                                     const float* x_token_scales, void* y, const void* w_sh,
                                     int32_t N2, float w_sh_scale,
                                     const float* w_sh_channel_scales, void* y_sh, void* ws,
                                     size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x || !ids || !y || !w_sh || !y_sh) return MOE_ERR_INVALID_ARG;
  if (p->desc.dtype != MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(w_sh) || !aligned16(y_sh) || N2 < 1 || N2 >= 65536 || N2 % 8)
    return MOE_ERR_INVALID_ARG;
  if (!p->side) {
    if (cudaStreamCreateWithFlags(&p->side, cudaStreamNonBlocking) != cudaSuccess)
      return MOE_ERR_CUDA;
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&p->sev[i], cudaEventDisableTiming) != cudaSuccess)
        return MOE_ERR_CUDA;
  }
  // fork: the shared expert on the plan's side stream, alongside the routed
  // path on `stream`; join before returning
  if (cudaEventRecord(p->sev[0], stream) != cudaSuccess ||
      cudaStreamWaitEvent(p->side, p->sev[0], 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  moe_status st = moe_shared_matmul(p, x, p->desc.N, p->desc.d, w_sh, N2, x_scale, x_token_scales,
                                    w_sh_scale, w_sh_channel_scales, y_sh, p->side);
  if (st != MOE_OK) return st;
  if (cudaEventRecord(p->sev[1], p->side) != cudaSuccess) return MOE_ERR_CUDA;
  st = moe_forward_routed(p, x, ids, gates, x_scale, x_token_scales, y, ws, ws_bytes, stream);
  if (cudaStreamWaitEvent(stream, p->sev[1], 0) != cudaSuccess) return MOE_ERR_CUDA;
  return st;
}

}  // extern "C"

namespace {
// The whole layer on n <= N tokens; every intermediate lives in the workspace.
moe_status forward_tokens(moe_plan p, int n, const void* x, void* y, void* ws, cudaStream_t stream) {
  const Layout& L = p->L;
  // decode-shaped bf16 SwiGLU batches: the gate/up GEMM gathers its rows from
  // x, the permute only makes the positions
  const bool gather = gather_fused(p->desc, n);
  moe_status st = run_router(p, n, x, at<int32_t>(ws, L.ids), at<float>(ws, L.gates), nullptr,
                             ws, stream);
  if (st == MOE_OK)
    st = run_permute(p, n, x, at<int32_t>(ws, L.ids), at<int32_t>(ws, L.counts),
                     at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.pos), at<int32_t>(ws, L.src),
                     gather ? nullptr : at<void>(ws, L.x_perm), ws, stream);
  if (st == MOE_OK)
    st = run_ffn(p, n, at<void>(ws, L.x_perm), at<int32_t>(ws, L.offsets), 1.f, nullptr, nullptr,
                 at<void>(ws, L.y_perm), ws, stream, nullptr, gather ? x : nullptr,
                 gather ? at<int32_t>(ws, L.src) : nullptr);
  if (st == MOE_OK)
    st = run_combine(p, n, at<void>(ws, L.y_perm), at<int32_t>(ws, L.pos), at<float>(ws, L.gates),
                     y, ws, stream);
  return st;
}

moe_status ensure_host_streams(moe_plan p) {
  if (p->h2d) return MOE_OK;
  if (cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking) != cudaSuccess)
    return MOE_ERR_CUDA;
  for (int i = 0; i < kHostEvents; ++i)
    if (cudaEventCreateWithFlags(&p->hev[i], cudaEventDisableTiming) != cudaSuccess)
      return MOE_ERR_CUDA;
  return MOE_OK;
}
}  // namespace

extern "C" {

moe_status moe_forward(moe_plan p, const void* x, void* y, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  if (!p || !x || !y || !p->w.w_r) return MOE_ERR_INVALID_ARG;
  if (!p->w.w1) return MOE_ERR_UNSUPPORTED;  // routing-only plan
  if (p->desc.dtype == MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.fwd_end);
  if (st != MOE_OK) return st;
  begin(p);
  st = forward_tokens(p, p->desc.N, x, y, ws, stream);
  end(p, stream);
  return st;
}

// Host buffers, asynchronous.  Staging slot s = call number % 2.  The H2D
// copy of x goes on a copy stream, after slot s was released by its previous
// user (two calls ago); the layer runs on the caller's stream once the copy
// landed; the D2H copy of y goes on a second copy stream once the layer is
// done, and then releases the slot.  Consecutive calls therefore overlap one
// batch's copies with the neighbouring batches' compute.
moe_status moe_forward_host_async(moe_plan p, const void* x_host, void* y_host, void* ws,
                                  size_t ws_bytes, moe_stream_t stream) {
  if (!p || !x_host || !y_host || !p->w.w_r) return MOE_ERR_INVALID_ARG;
  if (p->desc.dtype == MOE_E4M3 || !p->w.w1) return MOE_ERR_UNSUPPORTED;
  moe_status st = check_ws(p, ws, ws_bytes, p->L.total);
  if (st != MOE_OK) return st;
  if ((st = ensure_host_streams(p)) != MOE_OK) return st;
  const moe_layer_desc& d = p->desc;
  const int slot = static_cast<int>(p->host_calls & 1u);
  cudaEvent_t in_done = p->hev[3 * slot], out_ready = p->hev[3 * slot + 1],
              slot_free = p->hev[3 * slot + 2];
  char* xs = at<char>(ws, p->L.x_stage + slot * p->L.x_stage_bytes);
  char* ys = at<char>(ws, p->L.y_stage + slot * p->L.y_stage_bytes);
  const size_t xb = static_cast<size_t>(d.N) * d.d * p->ex;
  const size_t yb = static_cast<size_t>(d.N) * p->dout * p->ey;
  cudaStream_t cs = stream;
  if (p->host_calls >= 2 && cudaStreamWaitEvent(p->h2d, slot_free, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemcpyAsync(xs, x_host, xb, cudaMemcpyHostToDevice, p->h2d) != cudaSuccess ||
      cudaEventRecord(in_done, p->h2d) != cudaSuccess ||
      cudaStreamWaitEvent(cs, in_done, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  begin(p);
  st = forward_tokens(p, d.N, xs, ys, ws, cs);
  end(p, cs);
  if (st != MOE_OK) return st;
  if (cudaEventRecord(out_ready, cs) != cudaSuccess ||
      cudaStreamWaitEvent(p->d2h, out_ready, 0) != cudaSuccess ||
      cudaMemcpyAsync(y_host, ys, yb, cudaMemcpyDeviceToHost, p->d2h) != cudaSuccess ||
      cudaEventRecord(slot_free, p->d2h) != cudaSuccess)
    return MOE_ERR_CUDA;
  p->host_calls++;
  return MOE_OK;
}

moe_status moe_host_join(moe_plan p, moe_stream_t stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->h2d || p->host_calls == 0) return MOE_OK;
  const int last = static_cast<int>((p->host_calls - 1) & 1u);
  return cuda_status(cudaStreamWaitEvent(stream, p->hev[3 * last + 2], 0));
}

moe_status moe_forward_host(moe_plan p, const void* x_host, void* y_host, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
  moe_status st = moe_forward_host_async(p, x_host, y_host, ws, ws_bytes, stream);
  if (st != MOE_OK) return st;
  if ((st = moe_host_join(p, stream)) != MOE_OK) return st;
  return cuda_status(cudaStreamSynchronize(stream));
}

moe_status moe_read_device_status(moe_plan p, void* ws, moe_stream_t stream) {
  if (!p || !ws) return MOE_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpyAsync(&v, at<int>(ws, p->L.status), 4, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (v != 0) {
    if (cudaMemsetAsync(at<int>(ws, p->L.status), 0, 4, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return static_cast<moe_status>(v);
}

moe_status moe_profile_enable(moe_plan p, int enable) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (enable && !p->ev[0]) {
    for (int i = 0; i < kMaxEvents; ++i)
      if (cudaEventCreate(&p->ev[i]) != cudaSuccess) return MOE_ERR_CUDA;
  }
  p->profile = enable != 0;
  p->nev = 0;
  return MOE_OK;
}

moe_status moe_profile_read(moe_plan p, float* ms, const char** names, int capacity, int* count) {
  if (!p || !count) return MOE_ERR_INVALID_ARG;
  *count = 0;
  if (!p->profile || p->nev < 2) return MOE_OK;
  if (cudaEventSynchronize(p->ev[p->nev - 1]) != cudaSuccess) return MOE_ERR_CUDA;
  int n = 0;
  for (int i = 0; i + 1 < p->nev && n < capacity; ++i, ++n) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, p->ev[i], p->ev[i + 1]) != cudaSuccess) return MOE_ERR_CUDA;
    if (ms) ms[n] = t;
    if (names) names[n] = p->ev_name[i];
  }
  *count = n;
  return MOE_OK;
}

int moe_last_launch_count(moe_plan p) { return p ? p->launches : -1; }

}  // extern "C"

void moe::plan_call_begin(moe_plan_s* p) { begin(p); }
void moe::plan_call_mark(moe_plan_s* p, cudaStream_t s, const char* name_of_next) {
  mark(p, s, name_of_next);
}
void moe::plan_call_end(moe_plan_s* p, cudaStream_t s, int launches) {
  p->launches += launches;
  end(p, s);
}

bool moe::plan_permute_shape(const moe_plan_s* p, int* N, int* d, int* E, int* K,
                             int* row_bytes) {
  if (!p) return false;
  *N = p->desc.N;
  *d = p->desc.d;
  *E = p->desc.E;
  *K = p->desc.K;
  *row_bytes = p->desc.d * p->ex;
  return true;
}
