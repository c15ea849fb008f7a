// C ABI of the decode megakernel: handle creation, the decode step, status.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "mk_kernel.h"
#include "mk_plan.h"

static_assert(mk::kMaxTopK == MK_MAX_TOP_K, "the kernel's top-k bound is the ABI's");

using mk::KParams;
static_assert(sizeof(mk::TmaDesc) == sizeof(CUtensorMap), "TMA descriptor size");
using mk::LayerW;

struct mk_handle_s {
  mk_plan_s plan;
  int device = 0;
  KParams kp{};                 // everything but the per-step fields
  void* arena = nullptr;        // all device scratch in one allocation
  int* host_status = nullptr;   // mapped pinned word
  int32_t* h_stage = nullptr;   // pinned staging for the host-buffer step
  int32_t* d_stage = nullptr;   // device copy of token ids / positions / lengths
  float* d_logits = nullptr;    // device logits for the host-buffer step
  int32_t* d_argmax = nullptr;
  uint32_t epoch = 0;
  const void *kv_k = nullptr, *kv_v = nullptr;  // pools the KV tensor maps in kp were encoded for
  int32_t kv_pages = 0;
  std::string err;
};

static thread_local std::string g_err;
extern "C" const char* mk_internal_plan_error();

static int fail(mk_handle_t h, int code, const std::string& msg) {
  if (h) h->err = msg;
  else g_err = msg;
  return code;
}

static int cuda_fail(mk_handle_t h, cudaError_t e, const char* what) {
  return fail(h, MK_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define MK_CUDA(h, call)                                   \
  do {                                                     \
    cudaError_t e_ = (call);                               \
    if (e_ != cudaSuccess) return cuda_fail(h, e_, #call); \
  } while (0)

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static void release(mk_handle_t h) {
  if (!h) return;
  if (h->arena) cudaFree(h->arena);
  if (h->host_status) cudaFreeHost(h->host_status);
  if (h->h_stage) cudaFreeHost(h->h_stage);
  delete h;
}

// TMA descriptors of every weight matrix (bf16, 128-byte swizzle, boxes of 64 columns x
// 8n rows for n = 1..8).  wq/wk/wv are viewed as [heads*2 halves][head_dim/2][hidden]
// so that one box holds rows 8m..8m+8n-1 of both halves of a head (the RoPE pairs).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess && fn)
      encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
  }
  return encode;
}

static std::string build_tensor_maps(const mk_model_cfg& c, const mk_weight_ptrs* w, std::vector<CUtensorMap>& maps) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return "cuTensorMapEncodeTiled is not available";
  const mk::Geometry G = mk::geometry(c);
  maps.assign((size_t)mk::num_tmaps(G.L), CUtensorMap{});
  auto enc2d = [&](CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)mk::kBoxCols, box_rows};
    cuuint32_t es[2] = {1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  auto enc3d = [&](CUtensorMap* m, const void* ptr, uint64_t heads, uint32_t box_rows) {
    cuuint64_t dims[3] = {(cuuint64_t)G.d, (cuuint64_t)G.hd / 2, heads * 2};
    cuuint64_t strides[2] = {(cuuint64_t)G.d * 2, (cuuint64_t)(G.hd / 2) * G.d * 2};
    cuuint32_t box[3] = {(cuuint32_t)mk::kBoxCols, box_rows, 2};
    cuuint32_t es[3] = {1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  for (int l = 0; l < G.L; ++l) {
    for (int n = 1; n <= mk::kMaxBlocks; ++n) {
      const uint32_t br = 8u * n;
      CUresult r = CUDA_SUCCESS;
      if (n <= mk::max_units(mk::OP_QKV) && 8 * n <= G.hd / 2) {
        r = enc3d(&maps[mk::tmap_index(l, 0, n)], w->wq[l], G.nq, br);
        if (r == CUDA_SUCCESS) r = enc3d(&maps[mk::tmap_index(l, 1, n)], w->wk[l], G.nkv, br);
        if (r == CUDA_SUCCESS) r = enc3d(&maps[mk::tmap_index(l, 2, n)], w->wv[l], G.nkv, br);
      }
      if (r == CUDA_SUCCESS && n <= mk::max_units(mk::OP_GATEUP)) {
        r = enc2d(&maps[mk::tmap_index(l, 4, n)], w->w_gate[l], G.F, G.d, br);
        if (r == CUDA_SUCCESS) r = enc2d(&maps[mk::tmap_index(l, 5, n)], w->w_up[l], G.F, G.d, br);
      }
      if (r == CUDA_SUCCESS) r = enc2d(&maps[mk::tmap_index(l, 3, n)], w->wo[l], G.d, G.qdim, br);
      if (r == CUDA_SUCCESS) r = enc2d(&maps[mk::tmap_index(l, 6, n)], w->w_down[l], G.d, G.F, br);
      if (r != CUDA_SUCCESS) return "cuTensorMapEncodeTiled failed for layer " + std::to_string(l);
    }
  }
  for (int n = 1; n <= mk::kMaxBlocks; ++n)
    if (enc2d(&maps[mk::tmap_index(G.L, 0, n)], w->lm_head, G.V, G.d, 8u * n) != CUDA_SUCCESS)
      return "cuTensorMapEncodeTiled failed for the LM head";
  return "";
}

// Tensor maps of the GEMV operand buffers (appended after the weight maps): per operand kind,
// bf16 tile parts q = 2 * mt + part as rows of 64 values (boxes of 8 rows = 64 columns of one
// tile part), then the fp32 batch rows 0..kFmaRows-1 as lines of 32 values, ld / 32 lines per
// batch row (boxes of 2 lines = 64 columns).
static std::string encode_operand_maps(std::vector<CUtensorMap>& maps, int L, int ntiles,
                                       const __nv_bfloat16* const tiles[3], const float* const rows[3],
                                       const int lds[3]) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return "cuTensorMapEncodeTiled is not available";
  maps.resize((size_t)mk::num_all_tmaps(L), CUtensorMap{});
  cuuint32_t es[2] = {1, 1};
  for (int kind = 0; kind < 3; ++kind) {
    const int ld = lds[kind];
    for (int q = 0; q < 2 * ntiles; ++q) {
      cuuint64_t dims[2] = {64, (cuuint64_t)ld / 8};
      cuuint64_t strides[1] = {128};
      cuuint32_t box[2] = {64, 8};
      CUresult r = encode(&maps[mk::opmap_index(L, kind, q)], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<__nv_bfloat16*>(tiles[kind]) + (size_t)q * ld * 8, dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return "cuTensorMapEncodeTiled failed for an operand buffer";
    }
    cuuint64_t dims[2] = {32, (cuuint64_t)mk::kFmaRows * ld / 32};  // fp32 rows 0..kFmaRows-1, ld / 32 lines each
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {32, 2};
    CUresult r = encode(&maps[mk::opmap_index(L, kind, mk::kOpMapsPerKind - 1)], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                        const_cast<float*>(rows[kind]), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return "cuTensorMapEncodeTiled failed for an operand row";
  }
  return "";
}

// Tensor maps of the K and V pools, viewed as rows of head_dim values ([L][pages][nkv][16]
// rows): boxes of one 16-token page of one head with 128-byte swizzle.  head_dim 64: a 2-D
// box of 64 x 16; head_dim 128: a 3-D box {64 columns, 16 rows, 2 halves}, the halves
// outermost, so that each half of a page lands as 16 rows of 128 bytes.
static std::string encode_kv_maps(const mk_model_cfg& c, const mk_kv_cache* kv, KParams& k) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return "cuTensorMapEncodeTiled is not available";
  const uint64_t rows = (uint64_t)c.n_layers * (uint64_t)kv->num_pages * c.n_kv_heads * mk::kPage;
  if (rows >= (1ull << 31)) return "KV pool too large (layers * pages * kv heads * 16 must stay below 2^31)";
  void* pools[2] = {kv->k_pool, kv->v_pool};
  mk::TmaDesc* maps[2] = {&k.kmap, &k.vmap};
  for (int i = 0; i < 2; ++i) {
    CUresult r;
    cuuint32_t es[3] = {1, 1, 1};
    if (c.head_dim == 64) {
      cuuint64_t dims[2] = {64, rows};
      cuuint64_t strides[1] = {128};
      cuuint32_t box[2] = {64, (cuuint32_t)mk::kPage};
      r = encode(reinterpret_cast<CUtensorMap*>(maps[i]), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pools[i], dims,
                 strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
      cuuint64_t dims[3] = {64, rows, 2};
      cuuint64_t strides[2] = {256, 128};
      cuuint32_t box[3] = {64, (cuuint32_t)mk::kPage, 2};
      r = encode(reinterpret_cast<CUtensorMap*>(maps[i]), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, pools[i], dims,
                 strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return "cuTensorMapEncodeTiled failed for the KV pools (error " + std::to_string((int)r) + ")";
  }
  return "";
}

// ---------------------------------------------------------------------------------------
// Set-up shared by the handle (one cudaMalloc arena) and the allocation-free entry point (one
// __device__ array): weight checks, device checks, the scratch layout, the uploads and the
// kernel parameters.  Both paths lay the same pieces out in the same order.

// Check the weight pointers; collect the per-layer device pointers.  "" or an error message.
static std::string collect_layers(const mk_model_cfg& c, const mk_weight_ptrs* w, std::vector<LayerW>& lw) {
  if (!w->embed || !w->final_norm || !w->lm_head || !w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo ||
      !w->mlp_norm || !w->w_gate || !w->w_up || !w->w_down)
    return "null weight pointer";
  const void* all[3] = {w->embed, w->final_norm, w->lm_head};
  for (const void* p : all)
    if (!aligned16(p)) return "weights must be 16-byte aligned";
  lw.assign(c.n_layers > 0 ? c.n_layers : 0, LayerW{});
  for (int l = 0; l < c.n_layers; ++l) {
    const void* ps[9] = {w->attn_norm[l], w->wq[l], w->wk[l], w->wv[l], w->wo[l],
                         w->mlp_norm[l], w->w_gate[l], w->w_up[l], w->w_down[l]};
    for (const void* p : ps)
      if (!p || !aligned16(p)) return "layer weight null or not 16-byte aligned";
    lw[l] = LayerW{(const __nv_bfloat16*)ps[0], (const __nv_bfloat16*)ps[1], (const __nv_bfloat16*)ps[2],
                   (const __nv_bfloat16*)ps[3], (const __nv_bfloat16*)ps[4], (const __nv_bfloat16*)ps[5],
                   (const __nv_bfloat16*)ps[6], (const __nv_bfloat16*)ps[7], (const __nv_bfloat16*)ps[8],
                   nullptr, nullptr};
    if (c.qk_norm) {
      if (!w->q_norm || !w->k_norm) return "qk_norm needs the q_norm and k_norm arrays";
      const void* g[2] = {w->q_norm[l], w->k_norm[l]};
      for (const void* p : g)
        if (!p || !aligned16(p)) return "qk-norm gain null or not 16-byte aligned";
      lw[l].q_norm = (const __nv_bfloat16*)g[0];
      lw[l].k_norm = (const __nv_bfloat16*)g[1];
    }
  }
  return "";
}

// The device runs the kernel: sm_100, cooperative launch, enough threads.  MK_OK or a code
// with g_err set.
static int check_device(int dev, const char* who) {
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return fail(nullptr, MK_ERR_NO_DEVICE, "no CUDA device");
  if (prop.major != 10) return fail(nullptr, MK_ERR_NO_DEVICE, "the kernel is built for sm_100a (B200)");
  if (!prop.cooperativeLaunch) return fail(nullptr, MK_ERR_NO_DEVICE, "device lacks cooperative launch");
  int regs = 0, lmem = 0, maxthr = 0;
  cudaError_t ce = mk::kernel_attributes(&regs, &lmem, &maxthr);
  if (ce != cudaSuccess) return cuda_fail(nullptr, ce, "kernel attributes");
  if (maxthr < mk::kThreads)
    return fail(nullptr, MK_ERR_CUDA, std::string(who) + ": kernel cannot run its " + std::to_string(mk::kThreads) +
                                          " threads");
  return MK_OK;
}

// RoPE inverse frequencies, in double: theta^(-2j/hd), then the Llama-3.x frequency scaling
// when rope_scale_factor > 1 (the rule in mk.h's mk_model_cfg).
mk::RopeFreq mk_rope_freq(const mk_model_cfg& c) {
  mk::RopeFreq f{};
  const int half = c.head_dim / 2;
  const double pi = 3.14159265358979323846;
  for (int j = 0; j < half; ++j) {
    const double inv = std::pow((double)c.rope_theta, -2.0 * j / c.head_dim);
    double out = inv;
    if (c.rope_scale_factor > 1.f) {
      const double N = c.rope_original_max_pos, factor = c.rope_scale_factor;
      const double lo = c.rope_low_freq_factor, hi = c.rope_high_freq_factor;
      const double wavelen = 2.0 * pi / inv;
      if (wavelen > N / lo) {
        out = inv / factor;
      } else if (wavelen >= N / hi) {
        const double s = (N / wavelen - lo) / (hi - lo);
        out = (1.0 - s) * inv / factor + s * inv;
      }
    }
    f.inv_freq[j] = out;
  }
  return f;
}

// Byte offsets of the scratch pieces (256-byte aligned).  The last three serve only the
// handle's host-buffer entry point.
struct Layout {
  size_t layers, tasks, offs, maps, x, q, ax, aa, ah, ssq, part, lmpart, lmrows, spart, scnt, ctr, cmb, ctl, status,
      rope, qkss, knew;
  size_t stage, logits, argmax;
  size_t total;
  int ld_x, ld_a, ld_h, ntiles, ssq_stride, nsplit;
  std::vector<mk::TaskDesc> flat;   // the per-SM streams, concatenated
  std::vector<uint32_t> offs_host;  // per-SM offsets into flat
};

static Layout layout_scratch(const mk_plan_s& plan, bool host_step) {
  const mk_model_cfg& c = plan.cfg;
  const mk::Geometry G = mk::geometry(c);
  const int mb = c.max_batch;
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~size_t(255); return o; };
  L.offs_host.assign(plan.num_sms + 1, 0);
  for (int s = 0; s < plan.num_sms; ++s) {
    L.flat.insert(L.flat.end(), plan.streams[s].begin(), plan.streams[s].end());
    L.offs_host[s + 1] = (uint32_t)L.flat.size();
  }
  L.layers = take(sizeof(LayerW) * c.n_layers);
  L.tasks = take(sizeof(mk::TaskDesc) * L.flat.size());
  L.offs = take(sizeof(uint32_t) * L.offs_host.size());
  L.maps = take(sizeof(CUtensorMap) * (size_t)mk::num_all_tmaps(G.L));
  L.x = take(sizeof(float) * mb * G.d);
  L.q = take(sizeof(float) * mb * G.qdim);
  L.ld_x = mk::round_up(G.d, mk::kBoxCols);
  L.ld_a = mk::round_up(G.qdim, mk::kBoxCols);
  L.ld_h = mk::round_up(G.F, mk::kBoxCols);
  // operands: bf16 hi/lo tiles of 8 batch rows (opnd_tile_index layout) and fp32 batch rows
  // 0..kFmaRows-1, zero padded to whole 64-column boxes
  L.ntiles = (mb + 7) / 8;
  auto opbytes = [&](int ld) { return (size_t)L.ntiles * 2 * ld * 8 * 2 + (size_t)mk::kFmaRows * ld * 4; };
  L.ax = take(opbytes(L.ld_x));
  L.aa = take(opbytes(L.ld_a));
  L.ah = take(opbytes(L.ld_h));
  L.ssq_stride = plan.max_phase_tasks * mb;  // per instance: [task of the phase][max_b]
  L.ssq = take(sizeof(float) * (size_t)mk::num_ssq_inst(G.L) * L.ssq_stride);
  L.part = take(sizeof(float) * (size_t)mb * G.nkv * mk::kMaxChunksPerSeq * G.g * (G.hd + 2));
  L.lmpart = take(sizeof(float2) * (size_t)plan.n_lm_tasks * mb);
  L.lmrows = take(sizeof(int2) * (size_t)plan.n_lm_tasks);
  L.nsplit = plan.max_split_ids > 0 ? plan.max_split_ids : 1;
  L.spart = take(sizeof(float) * (size_t)L.nsplit * mk::kMaxPieces * mk::kMaxBlocks * 8 * mb);
  L.scnt = take(sizeof(uint32_t) * (size_t)L.nsplit);
  L.ctr = take(sizeof(uint32_t) * mk::num_counters(G.L));
  L.cmb = take(sizeof(uint32_t) * (size_t)G.L * mb * G.nkv);
  L.ctl = take(sizeof(uint32_t) * 2);
  L.status = take(sizeof(int));
  L.rope = take(sizeof(float2) * (size_t)c.max_ctx * (G.hd / 2));
  L.qkss = L.knew = 0;
  if (c.qk_norm) {
    L.qkss = take(sizeof(float) * (size_t)mb * (G.nq + G.nkv) * (G.hd / 16));
    L.knew = take(sizeof(float) * (size_t)mb * G.nkv * G.hd);
  }
  L.stage = L.logits = L.argmax = 0;
  if (host_step) {
    L.stage = take(sizeof(int32_t) * 3 * mb);
    L.logits = take(sizeof(float) * (size_t)mb * G.V);
    L.argmax = take(sizeof(int32_t) * mb);
  }
  L.total = off;
  return L;
}

// Encode the tensor maps of (plan, weights) for scratch at `A`, clear the scratch, upload the
// tables and compute the RoPE table, in order on `stream`, then synchronise it.
static int upload_tables(const mk_plan_s& plan, const mk_weight_ptrs* w, const std::vector<LayerW>& lw,
                         const Layout& L, unsigned char* A, cudaStream_t stream, const char* who) {
  const mk_model_cfg& c = plan.cfg;
  const mk::Geometry G = mk::geometry(c);
  std::vector<CUtensorMap> maps;
  std::string merr = build_tensor_maps(c, w, maps);
  if (merr.empty()) {
    auto tl = [&](size_t o) { return (const __nv_bfloat16*)(A + o); };
    auto rw = [&](size_t o, int ld) { return (const float*)(A + o + (size_t)L.ntiles * 2 * ld * 8 * 2); };
    const __nv_bfloat16* tiles[3] = {tl(L.ax), tl(L.aa), tl(L.ah)};
    const float* rows[3] = {rw(L.ax, L.ld_x), rw(L.aa, L.ld_a), rw(L.ah, L.ld_h)};
    const int lds[3] = {L.ld_x, L.ld_a, L.ld_h};
    merr = encode_operand_maps(maps, G.L, L.ntiles, tiles, rows, lds);
  }
  if (!merr.empty()) return fail(nullptr, MK_ERR_CUDA, std::string(who) + ": " + merr);
  cudaError_t ce = cudaMemsetAsync(A, 0, L.total, stream);
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(A + L.layers, lw.data(), sizeof(LayerW) * c.n_layers, cudaMemcpyHostToDevice, stream);
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(A + L.tasks, L.flat.data(), sizeof(mk::TaskDesc) * L.flat.size(), cudaMemcpyHostToDevice,
                         stream);
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(A + L.offs, L.offs_host.data(), sizeof(uint32_t) * L.offs_host.size(),
                         cudaMemcpyHostToDevice, stream);
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(A + L.maps, maps.data(), sizeof(CUtensorMap) * maps.size(), cudaMemcpyHostToDevice, stream);
  if (ce == cudaSuccess) ce = mk::launch_rope_table((float2*)(A + L.rope), c.max_ctx, G.hd, mk_rope_freq(c), stream);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(stream);
  if (ce != cudaSuccess) return cuda_fail(nullptr, ce, (std::string(who) + ": upload").c_str());
  return MK_OK;
}

// Kernel parameters (all but the per-step fields) of a plan laid out at `A`.
static KParams make_kparams(const mk_plan_s& plan, const mk_weight_ptrs* w, const Layout& L, unsigned char* A,
                            int* status) {
  const mk_model_cfg& c = plan.cfg;
  const mk::Geometry G = mk::geometry(c);
  KParams k{};
  k.L = G.L; k.d = G.d; k.nq = G.nq; k.nkv = G.nkv; k.hd = G.hd; k.F = G.F; k.V = G.V; k.g = G.g;
  k.qdim = G.qdim; k.max_b = c.max_batch; k.max_ctx = c.max_ctx; k.eps = c.rms_eps;
  k.layers = (const LayerW*)(A + L.layers);
  k.embed = (const __nv_bfloat16*)w->embed;
  k.final_norm = (const __nv_bfloat16*)w->final_norm;
  k.lm_head = (const __nv_bfloat16*)w->lm_head;
  k.tasks = (const mk::TaskDesc*)(A + L.tasks);
  k.task_off = (const uint32_t*)(A + L.offs);
  k.num_sms = plan.num_sms;
  k.n_slots = plan.num_sms * plan.attn_slots_per_sm;
  k.n_lm_tasks = plan.n_lm_tasks;
  k.tmaps = A + L.maps;
  k.x = (float*)(A + L.x);
  k.q = (float*)(A + L.q);
  auto carve = [&](size_t o, int ld, __nv_bfloat16** t, float** f) {
    *t = (__nv_bfloat16*)(A + o);
    *f = (float*)(*t + (size_t)L.ntiles * 2 * ld * 8);
  };
  carve(L.ax, L.ld_x, &k.ax_t, &k.ax_f);
  carve(L.aa, L.ld_a, &k.aa_t, &k.aa_f);
  carve(L.ah, L.ld_h, &k.ah_t, &k.ah_f);
  k.ld_x = L.ld_x; k.ld_a = L.ld_a; k.ld_h = L.ld_h;
  k.ssq = (float*)(A + L.ssq);
  k.ssq_stride = L.ssq_stride;
  k.part = (float*)(A + L.part);
  k.lmpart = (float2*)(A + L.lmpart);
  k.lmrows = (int2*)(A + L.lmrows);
  k.qk_norm = c.qk_norm ? 1 : 0;
  k.qkss = c.qk_norm ? (float*)(A + L.qkss) : nullptr;
  k.knew = c.qk_norm ? (float*)(A + L.knew) : nullptr;
  k.spart = (float*)(A + L.spart);
  k.scnt = (uint32_t*)(A + L.scnt);
  k.n_split = L.nsplit;
  k.ctr = (uint32_t*)(A + L.ctr);
  k.cmb = (uint32_t*)(A + L.cmb);
  k.ctl = (uint32_t*)(A + L.ctl);
  k.host_status = status;
  k.rope = (const float2*)(A + L.rope);
  k.timeout_ns = 1000000000ull;
  k.dbg = nullptr;
  k.trace = nullptr;
  return k;
}

// Zero what the kernel expects at zero after a failed step: dependency, combine and K-piece
// counters, the abort flag and first error code.
static cudaError_t clear_counters(const KParams& k, cudaStream_t s) {
  cudaError_t ce = cudaMemsetAsync(k.ctr, 0, sizeof(uint32_t) * mk::num_counters(k.L), s);
  if (ce == cudaSuccess) ce = cudaMemsetAsync(k.cmb, 0, sizeof(uint32_t) * (size_t)k.L * k.max_b * k.nkv, s);
  if (ce == cudaSuccess) ce = cudaMemsetAsync(k.ctl, 0, sizeof(uint32_t) * 2, s);
  if (ce == cudaSuccess) ce = cudaMemsetAsync(k.scnt, 0, sizeof(uint32_t) * (size_t)k.n_split, s);
  return ce;
}

extern "C" {

MK_API int mk_create_from_plan(mk_plan_t plan, const mk_weight_ptrs* w, int32_t flags, mk_handle_t* out) {
  if (!plan || !w || !out) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_create: null argument");
  const mk_model_cfg& c = plan->cfg;
  std::string e;
  if (!(flags & MK_CREATE_SKIP_VALIDATE)) {
    int rc = mk::validate_plan(*plan, &e);
    if (rc) return fail(nullptr, rc, "schedule rejected: " + e);
  }
  std::vector<LayerW> lw;
  e = collect_layers(c, w, lw);
  if (!e.empty()) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_create: " + e);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(nullptr, MK_ERR_NO_DEVICE, "no CUDA device");
  int rc = check_device(dev, "mk_create");
  if (rc) return rc;
  int nsm = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (plan->num_sms != nsm)
    return fail(nullptr, MK_ERR_INVALID_ARG,
                "plan built for " + std::to_string(plan->num_sms) + " SMs, device has " + std::to_string(nsm));

  mk_handle_t h = new mk_handle_s();
  h->plan = *plan;
  h->device = dev;
  const Layout L = layout_scratch(*plan, true);
  cudaError_t ce = cudaMalloc(&h->arena, L.total);
  if (ce == cudaSuccess) ce = cudaHostAlloc((void**)&h->host_status, sizeof(int), cudaHostAllocMapped);
  if (ce == cudaSuccess) ce = cudaHostAlloc((void**)&h->h_stage, sizeof(int32_t) * 3 * c.max_batch, cudaHostAllocDefault);
  if (ce != cudaSuccess) { release(h); return cuda_fail(nullptr, ce, "scratch allocation"); }
  *h->host_status = 0;
  int* dev_status = nullptr;
  ce = cudaHostGetDevicePointer((void**)&dev_status, h->host_status, 0);
  if (ce != cudaSuccess) { release(h); return cuda_fail(nullptr, ce, "cudaHostGetDevicePointer"); }
  unsigned char* A = (unsigned char*)h->arena;
  rc = upload_tables(*plan, w, lw, L, A, 0, "mk_create");
  if (rc) { release(h); return rc; }
  h->kp = make_kparams(*plan, w, L, A, dev_status);
  h->d_stage = (int32_t*)(A + L.stage);
  h->d_logits = (float*)(A + L.logits);
  h->d_argmax = (int32_t*)(A + L.argmax);
  h->err.clear();
  *out = h;
  return MK_OK;
}

MK_API int mk_create(const mk_model_cfg* cfg, const mk_weight_ptrs* w, mk_handle_t* out) {
  if (!cfg || !w || !out) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_create: null argument");
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(nullptr, MK_ERR_NO_DEVICE, "no CUDA device");
  mk_plan_opts o{};
  o.num_sms = nsm;
  mk_plan_t plan = nullptr;
  int rc = mk_plan_create(cfg, &o, &plan);
  if (rc) return fail(nullptr, rc, std::string("plan: ") + mk_internal_plan_error());
  rc = mk_create_from_plan(plan, w, 0, out);
  mk_plan_destroy(plan);
  return rc;
}

static int check_step_args(mk_handle_t h, const void* tok, const void* pos, const void* lens, int32_t batch,
                           const mk_kv_cache* kv, const void* logits) {
  const mk_model_cfg& c = h->plan.cfg;
  if (!tok || !pos || !lens || !kv || !logits) return fail(h, MK_ERR_INVALID_ARG, "mk_decode_step: null argument");
  if (batch < 1 || batch > c.max_batch)
    return fail(h, MK_ERR_INVALID_ARG, "mk_decode_step: batch must be in [1, max_batch]");
  if (!kv->k_pool || !kv->v_pool || !kv->page_table || kv->num_pages < 1 || kv->max_pages_per_seq < 1)
    return fail(h, MK_ERR_INVALID_ARG, "mk_decode_step: bad kv cache description");
  if (!aligned16(kv->k_pool) || !aligned16(kv->v_pool))
    return fail(h, MK_ERR_INVALID_ARG, "mk_decode_step: kv pools must be 16-byte aligned");
  int st = *(volatile int*)h->host_status;
  if (st != 0) return fail(h, st, "mk_decode_step: a previous step failed on the device; call mk_reset");
  return MK_OK;
}

static int launch_step(mk_handle_t h, const int32_t* tok, const int32_t* pos, const int32_t* lens, int32_t batch,
                       const mk_kv_cache* kv, float* logits, int32_t* argmax, cudaStream_t s, int step_add = 0,
                       const mk_sampling* smp = nullptr, const float* uniforms = nullptr,
                       const int32_t* group_first = nullptr) {
  if (kv->k_pool != h->kv_k || kv->v_pool != h->kv_v || kv->num_pages != h->kv_pages) {
    const std::string e = encode_kv_maps(h->plan.cfg, kv, h->kp);
    if (!e.empty()) {
      h->kv_k = h->kv_v = nullptr;
      return fail(h, MK_ERR_INVALID_ARG, "mk_decode_step: " + e);
    }
    h->kv_k = kv->k_pool;
    h->kv_v = kv->v_pool;
    h->kv_pages = kv->num_pages;
  }
  KParams p = h->kp;
  p.tok = tok; p.pos = pos; p.lens = lens; p.b = batch; p.step_add = step_add;
  p.group_first = group_first;
  p.kpool = (__nv_bfloat16*)kv->k_pool; p.vpool = (__nv_bfloat16*)kv->v_pool;
  p.ptable = kv->page_table; p.num_pages = kv->num_pages; p.mpps = kv->max_pages_per_seq;
  p.logits = logits; p.argmax = argmax;
  if (smp && smp->top_k > 1) {
    p.top_k = smp->top_k;
    p.temperature = smp->temperature;
    p.uniforms = uniforms;
  }
  p.epoch = ++h->epoch;
  cudaError_t e = mk::launch_decode(p, s);
  if (e != cudaSuccess) {
    --h->epoch;
    return cuda_fail(h, e, "megakernel launch");
  }
  return MK_OK;
}

MK_API int mk_decode_step(mk_handle_t h, const int32_t* token_ids, const int32_t* positions,
                          const int32_t* seq_lens, int32_t batch, const mk_kv_cache* kv, float* logits_out,
                          int32_t* argmax_out, mk_stream_t stream) {
  if (!h) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step: null handle");
  int rc = check_step_args(h, token_ids, positions, seq_lens, batch, kv, logits_out);
  if (rc) return rc;
  return launch_step(h, token_ids, positions, seq_lens, batch, kv, logits_out, argmax_out, (cudaStream_t)stream);
}

MK_API int mk_decode_steps(mk_handle_t h, int32_t n_steps, const int32_t* token_ids, const int32_t* positions,
                           int32_t batch, const mk_kv_cache* kv, const mk_sampling* sampling, int32_t* tokens_out,
                           float* logits_out, mk_stream_t stream) {
  if (!h) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_steps: null handle");
  if (n_steps < 1) return fail(h, MK_ERR_INVALID_ARG, "mk_decode_steps: n_steps must be >= 1");
  if (!tokens_out) return fail(h, MK_ERR_INVALID_ARG, "mk_decode_steps: null tokens_out");
  if (sampling && sampling->top_k > 1) {
    if (sampling->top_k > MK_MAX_TOP_K)
      return fail(h, MK_ERR_INVALID_ARG, "mk_decode_steps: top_k above MK_MAX_TOP_K");
    if (!(sampling->temperature > 0.f) || !std::isfinite(sampling->temperature))
      return fail(h, MK_ERR_INVALID_ARG, "mk_decode_steps: temperature must be finite and > 0");
    if (!sampling->uniforms) return fail(h, MK_ERR_INVALID_ARG, "mk_decode_steps: null uniforms");
  }
  float* logits = logits_out ? logits_out : h->d_logits;
  int rc = check_step_args(h, token_ids, positions, positions, batch, kv, logits);
  if (rc) return rc;
  const cudaStream_t s = (cudaStream_t)stream;
  for (int32_t k = 0; k < n_steps; ++k) {
    // step k: the token is step k-1's greedy token, every position k further on
    const int32_t* tok = k == 0 ? token_ids : tokens_out + (size_t)(k - 1) * batch;
    rc = launch_step(h, tok, positions, nullptr, batch, kv, logits, tokens_out + (size_t)k * batch, s, k, sampling,
                     sampling ? sampling->uniforms + (size_t)k * batch : nullptr);
    if (rc) return rc;
  }
  return MK_OK;
}

MK_API int mk_verify_step(mk_handle_t h, const int32_t* token_ids, const int32_t* positions,
                          const int32_t* seq_lens, const int32_t* group_first, int32_t batch, const mk_kv_cache* kv,
                          float* logits_out, int32_t* argmax_out, mk_stream_t stream) {
  if (!h) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_verify_step: null handle");
  if (!group_first) return fail(h, MK_ERR_INVALID_ARG, "mk_verify_step: null group_first");
  int rc = check_step_args(h, token_ids, positions, seq_lens, batch, kv, logits_out);
  if (rc) return rc;
  return launch_step(h, token_ids, positions, seq_lens, batch, kv, logits_out, argmax_out, (cudaStream_t)stream, 0,
                     nullptr, nullptr, group_first);
}

MK_API int mk_decode_step_host(mk_handle_t h, const int32_t* token_ids, const int32_t* positions,
                               const int32_t* seq_lens, int32_t batch, const mk_kv_cache* kv, float* logits_host,
                               int32_t* argmax_host, mk_stream_t stream) {
  if (!h) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step_host: null handle");
  int rc = check_step_args(h, token_ids, positions, seq_lens, batch, kv, h->d_logits);
  if (rc) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  const int mb = h->plan.cfg.max_batch;
  // one pinned staging buffer -> one H2D copy of the three int arrays
  std::memcpy(h->h_stage, token_ids, sizeof(int32_t) * batch);
  std::memcpy(h->h_stage + mb, positions, sizeof(int32_t) * batch);
  std::memcpy(h->h_stage + 2 * mb, seq_lens, sizeof(int32_t) * batch);
  MK_CUDA(h, cudaMemcpyAsync(h->d_stage, h->h_stage, sizeof(int32_t) * 3 * mb, cudaMemcpyHostToDevice, s));
  rc = launch_step(h, h->d_stage, h->d_stage + mb, h->d_stage + 2 * mb, batch, kv, h->d_logits,
                   argmax_host ? h->d_argmax : nullptr, s);
  if (rc) return rc;
  const size_t V = (size_t)h->plan.cfg.vocab;
  if (logits_host)
    MK_CUDA(h, cudaMemcpyAsync(logits_host, h->d_logits, sizeof(float) * V * batch, cudaMemcpyDeviceToHost, s));
  if (argmax_host)
    MK_CUDA(h, cudaMemcpyAsync(argmax_host, h->d_argmax, sizeof(int32_t) * batch, cudaMemcpyDeviceToHost, s));
  MK_CUDA(h, cudaStreamSynchronize(s));
  int st = *(volatile int*)h->host_status;
  if (st != 0) return fail(h, st, "mk_decode_step_host: the step failed on the device");
  return MK_OK;
}

MK_API int mk_get_status(mk_handle_t h) {
  if (!h) return MK_ERR_INVALID_ARG;
  return *(volatile int*)h->host_status;
}

MK_API int mk_reset(mk_handle_t h) {
  if (!h) return MK_ERR_INVALID_ARG;
  MK_CUDA(h, cudaDeviceSynchronize());
  MK_CUDA(h, clear_counters(h->kp, 0));
  MK_CUDA(h, cudaDeviceSynchronize());
  *(volatile int*)h->host_status = 0;
  h->epoch = 0;
  return MK_OK;
}

MK_API int mk_set_debug(mk_handle_t h, float* layer_hidden) {
  if (!h) return MK_ERR_INVALID_ARG;
  h->kp.dbg = layer_hidden;
  return MK_OK;
}

MK_API int mk_set_trace(mk_handle_t h, uint64_t* records, int64_t capacity) {
  if (!h) return MK_ERR_INVALID_ARG;
  int64_t n = 0;
  for (const auto& s : h->plan.streams) n += (int64_t)s.size();
  if (records && capacity < n) return fail(h, MK_ERR_INVALID_ARG, "mk_set_trace: capacity below the task count");
  h->kp.trace = (unsigned long long*)records;
  return MK_OK;
}

MK_API int64_t mk_num_tasks(mk_handle_t h) {
  if (!h) return MK_ERR_INVALID_ARG;
  int64_t n = 0;
  for (const auto& s : h->plan.streams) n += (int64_t)s.size();
  return n;
}

MK_API int mk_set_timeout_ns(mk_handle_t h, uint64_t ns) {
  if (!h || ns == 0) return MK_ERR_INVALID_ARG;
  h->kp.timeout_ns = ns;
  return MK_OK;
}

MK_API int mk_launches_per_step(mk_handle_t h) { return h ? 1 : MK_ERR_INVALID_ARG; }

MK_API int mk_destroy(mk_handle_t h) {
  if (!h) return MK_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  release(h);
  return MK_OK;
}

MK_API const char* mk_last_error(mk_handle_t h) { return h ? h->err.c_str() : g_err.c_str(); }

MK_API int mk_route_pick(const int32_t* max_batch, const int32_t* max_ctx, int32_t n, int32_t batch,
                         int32_t max_position) {
  if (!max_batch || !max_ctx || n < 1 || batch < 1 || max_position < 0) return MK_ERR_INVALID_ARG;
  int best = -1;
  for (int i = 0; i < n; ++i) {
    if (max_batch[i] < batch || max_ctx[i] <= max_position) continue;
    if (best < 0 || max_batch[i] < max_batch[best] ||
        (max_batch[i] == max_batch[best] && max_ctx[i] < max_ctx[best]))
      best = i;
  }
  return best < 0 ? MK_ERR_INVALID_ARG : best;
}

struct mk_router_s {
  std::vector<mk_handle_t> handles;
  std::vector<int32_t> max_batch, max_ctx;
};

MK_API int mk_router_create(const mk_handle_t* handles, int32_t n, mk_router_t* out) {
  if (!handles || n < 1 || !out) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_router_create: bad arguments");
  mk_router_t r = new mk_router_s();
  for (int i = 0; i < n; ++i) {
    if (!handles[i]) { delete r; return fail(nullptr, MK_ERR_INVALID_ARG, "mk_router_create: null handle"); }
    const mk_model_cfg& c = handles[i]->plan.cfg;
    const mk_model_cfg& c0 = handles[0]->plan.cfg;
    if (c.n_layers != c0.n_layers || c.hidden != c0.hidden || c.vocab != c0.vocab || c.n_heads != c0.n_heads ||
        c.n_kv_heads != c0.n_kv_heads || c.head_dim != c0.head_dim || c.ffn != c0.ffn) {
      delete r;
      return fail(nullptr, MK_ERR_INVALID_ARG, "mk_router_create: handles of different models");
    }
    r->handles.push_back(handles[i]);
    r->max_batch.push_back(c.max_batch);
    r->max_ctx.push_back(c.max_ctx);
  }
  *out = r;
  return MK_OK;
}

MK_API int mk_router_step(mk_router_t r, const int32_t* token_ids, const int32_t* positions, const int32_t* seq_lens,
                          int32_t batch, int32_t max_position, const mk_kv_cache* kv, float* logits_out,
                          int32_t* argmax_out, int32_t* picked, mk_stream_t stream) {
  if (!r) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_router_step: null router");
  const int i = mk_route_pick(r->max_batch.data(), r->max_ctx.data(), (int32_t)r->handles.size(), batch,
                              max_position);
  if (i < 0) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_router_step: no handle covers this batch and position");
  if (picked) *picked = i;
  return mk_decode_step(r->handles[i], token_ids, positions, seq_lens, batch, kv, logits_out, argmax_out, stream);
}

MK_API int mk_router_destroy(mk_router_t r) {
  if (!r) return MK_ERR_INVALID_ARG;
  delete r;
  return MK_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// The decode step on statically allocated scratch.
//
// For callers that may not allocate device memory: a process whose HBM belongs to another
// allocator (a caching allocator that has reserved the free memory, where a cudaMalloc
// beside it fails or fragments the pool), or a latency-critical serving loop in which a
// cudaMalloc/cudaFree would synchronise the device.  The scratch the megakernel needs
// (task streams, tensor maps, activations, partial sums, dependency counters, RoPE table,
// status word) is carved from one file-scope __device__ array instead of a handle's
// cudaMalloc arena; the kernel and its launch are the ones mk_decode_step uses.

#include <mutex>

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // the most one device's tables may take
constexpr int kStaticMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct StaticState {
  unsigned char* base = nullptr;   // device address of g_static_scratch on this device
  bool ready = false;              // the tables below were uploaded for cfg/weights
  bool dirty = false;              // counters and status must be cleared before the next launch
  mk_model_cfg cfg{};
  std::vector<const void*> wkey;   // the weight pointers the tables were built for
  KParams kp{};
  int* status = nullptr;           // device word the kernel reports a failure in
  uint32_t epoch = 0;
  const void *kv_k = nullptr, *kv_v = nullptr;  // pools the KV tensor maps in kp were encoded for
  int32_t kv_pages = 0;
};

StaticState g_static[kStaticMaxDevices];
std::mutex g_static_mu[kStaticMaxDevices];

void weight_key(const mk_model_cfg& c, const mk_weight_ptrs* w, std::vector<const void*>* out) {
  out->assign({w->embed, w->final_norm, w->lm_head});
  const void* const* per[11] = {w->attn_norm, w->wq, w->wk, w->wv, w->wo, w->mlp_norm, w->w_gate, w->w_up,
                                 w->w_down, c.qk_norm ? w->q_norm : nullptr, c.qk_norm ? w->k_norm : nullptr};
  for (const void* const* a : per)
    for (int l = 0; l < c.n_layers; ++l) out->push_back(a ? a[l] : nullptr);
}

bool same_key(const StaticState& s, const mk_model_cfg& c, const mk_weight_ptrs* w) {
  if (!s.ready || std::memcmp(&s.cfg, &c, sizeof(c)) != 0) return false;
  const void* head[3] = {w->embed, w->final_norm, w->lm_head};
  for (int i = 0; i < 3; ++i)
    if (s.wkey[i] != head[i]) return false;
  const void* const* per[11] = {w->attn_norm, w->wq, w->wk, w->wv, w->wo, w->mlp_norm, w->w_gate, w->w_up,
                                 w->w_down, c.qk_norm ? w->q_norm : nullptr, c.qk_norm ? w->k_norm : nullptr};
  size_t k = 3;
  for (int a = 0; a < 11; ++a)
    for (int l = 0; l < c.n_layers; ++l, ++k)
      if ((per[a] ? per[a][l] : nullptr) != s.wkey[k]) return false;
  return true;
}

// Build the schedule and tensor maps for (cfg, weights), lay the scratch out in the static
// array (the same layout as a handle's arena, without the host-buffer pieces), clear it and
// upload the tables.  Host-synchronous on `stream`.
int static_setup(StaticState& s, const mk_model_cfg& c, const mk_weight_ptrs* w, int dev, cudaStream_t stream) {
  s.ready = false;
  std::vector<LayerW> lw;
  const std::string e = collect_layers(c, w, lw);
  if (!e.empty()) return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step_static: " + e);
  int rc = check_device(dev, "mk_decode_step_static");
  if (rc) return rc;
  mk_plan_opts o{};
  cudaDeviceGetAttribute(&o.num_sms, cudaDevAttrMultiProcessorCount, dev);
  mk_plan_s plan;
  std::string pe;
  rc = mk::build_plan(c, &o, &plan, &pe);
  if (rc) return fail(nullptr, rc, "plan: " + pe);
  rc = mk::validate_plan(plan, &pe);
  if (rc) return fail(nullptr, rc, "schedule rejected: " + pe);
  const Layout L = layout_scratch(plan, false);
  if (L.total > kStaticScratchBytes)
    return fail(nullptr, MK_ERR_INVALID_ARG,
                "mk_decode_step_static: this model needs " + std::to_string(L.total) +
                    " bytes of scratch; the static area holds " + std::to_string(kStaticScratchBytes) +
                    " (lower max_batch or max_ctx, or use mk_create)");
  rc = upload_tables(plan, w, lw, L, s.base, stream, "mk_decode_step_static");
  if (rc) return rc;
  s.kp = make_kparams(plan, w, L, s.base, (int*)(s.base + L.status));
  s.kv_k = s.kv_v = nullptr;
  s.status = (int*)(s.base + L.status);
  s.cfg = c;
  weight_key(c, w, &s.wkey);
  s.epoch = 0;
  s.dirty = false;
  s.ready = true;
  return MK_OK;
}

// Zero what the kernel expects to start at zero after a failed step: the counters, the abort
// flag and first error code, the status word.
cudaError_t static_clear(StaticState& s, cudaStream_t stream) {
  cudaError_t ce = clear_counters(s.kp, stream);
  if (ce == cudaSuccess) ce = cudaMemsetAsync(s.status, 0, sizeof(int), stream);
  return ce;
}

}  // namespace

extern "C" MK_API int mk_decode_step_static(const mk_model_cfg* cfg, const mk_weight_ptrs* weights,
                                            const int32_t* token_ids, const int32_t* positions,
                                            const int32_t* seq_lens, int32_t batch, const mk_kv_cache* kv,
                                            float* logits_out, int32_t* argmax_out, mk_stream_t stream) {
  if (!cfg || !weights || !token_ids || !positions || !seq_lens || !kv || !logits_out)
    return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step_static: null argument");
  if (batch < 1 || batch > cfg->max_batch)
    return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step_static: batch must be in [1, max_batch]");
  if (!kv->k_pool || !kv->v_pool || !kv->page_table || kv->num_pages < 1 || kv->max_pages_per_seq < 1)
    return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step_static: bad kv cache description");
  if (!aligned16(kv->k_pool) || !aligned16(kv->v_pool))
    return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step_static: kv pools must be 16-byte aligned");
  std::string cerr;
  int rc = mk::check_cfg(*cfg, &cerr);
  if (rc) return fail(nullptr, rc, "mk_decode_step_static: " + cerr);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(nullptr, MK_ERR_NO_DEVICE, "no CUDA device");
  if (dev < 0 || dev >= kStaticMaxDevices)
    return fail(nullptr, MK_ERR_NO_DEVICE, "mk_decode_step_static: device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_static_mu[dev]);
  StaticState& s = g_static[dev];
  cudaStream_t st = (cudaStream_t)stream;
  {
    // the address of this device's copy of the array, looked up with the device current on every
    // call (it is cheap): if the module was loaded anew (after a device reset), the tables are
    // gone and the set-up runs again
    void* p = nullptr;
    cudaError_t ce = cudaGetSymbolAddress(&p, g_static_scratch);
    if (ce != cudaSuccess) return cuda_fail(nullptr, ce, "mk_decode_step_static: cudaGetSymbolAddress");
    if ((unsigned char*)p != s.base) {
      s.base = (unsigned char*)p;
      s.ready = false;
    }
  }
  if (!same_key(s, *cfg, weights)) {
    rc = static_setup(s, *cfg, weights, dev, st);
    if (rc) return rc;
  }
  if (s.dirty) {
    cudaError_t ce = static_clear(s, st);
    if (ce != cudaSuccess) return cuda_fail(nullptr, ce, "mk_decode_step_static: clear");
    s.epoch = 0;
    s.dirty = false;
  }
  if (kv->k_pool != s.kv_k || kv->v_pool != s.kv_v || kv->num_pages != s.kv_pages) {
    const std::string e = encode_kv_maps(*cfg, kv, s.kp);
    if (!e.empty()) {
      s.kv_k = s.kv_v = nullptr;
      return fail(nullptr, MK_ERR_INVALID_ARG, "mk_decode_step_static: " + e);
    }
    s.kv_k = kv->k_pool;
    s.kv_v = kv->v_pool;
    s.kv_pages = kv->num_pages;
  }
  KParams p = s.kp;
  p.tok = token_ids; p.pos = positions; p.lens = seq_lens; p.b = batch;
  p.kpool = (__nv_bfloat16*)kv->k_pool; p.vpool = (__nv_bfloat16*)kv->v_pool;
  p.ptable = kv->page_table; p.num_pages = kv->num_pages; p.mpps = kv->max_pages_per_seq;
  p.logits = logits_out; p.argmax = argmax_out;
  p.epoch = ++s.epoch;
  cudaError_t ce = mk::launch_decode(p, st);
  if (ce != cudaSuccess) {
    --s.epoch;
    return cuda_fail(nullptr, ce, "mk_decode_step_static: megakernel launch");
  }
  int status = 0;
  ce = cudaMemcpyAsync(&status, s.status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  if (ce != cudaSuccess) {
    s.dirty = true;
    return cuda_fail(nullptr, ce, "mk_decode_step_static: step");
  }
  if (status != 0) {
    s.dirty = true;
    return fail(nullptr, status, "mk_decode_step_static: the step failed on the device");
  }
  return MK_OK;
}
