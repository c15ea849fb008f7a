// The kernel-per-op decode step: the same Llama-style step as the megakernel, run the way
// a conventional engine runs it - one launch per operation, 10 per layer plus 4 - replayed
// as a CUDA graph whose launches carry programmatic dependent launch (each kernel's launch
// and prologue may start while its predecessor finishes; it waits for the predecessor's
// results with griddepcontrol.wait).
//
// It exists to measure what the single-launch design removes: launches per token, the
// device time they add between kernels, and the synchronisation at every kernel boundary
// ("ForgeMegakernel" §1: engines launch 280-448 kernels per token, and kernel start-up and
// retirement make decoding take 1.06-1.45x as long as one persistent kernel moving the same
// bytes; §2.3 "Megakernels").  The kernels are plain CUDA-core code (fp32 arithmetic on bf16
// weights and cache); batches up to 8, head_dim 64 or 128, no QK-norm.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "mk_kernel.h"
#include "mk_plan.h"

using bf16 = __nv_bfloat16;

namespace kpo {

constexpr int kMaxB = 8;         // largest batch
constexpr int kChunk = 256;      // keys per attention block (split-K)

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// x[bi][c] = E[tok[bi]][c]
// (a token id outside the vocabulary gives a NaN row instead of a read out of bounds)
__global__ void embed_k(const bf16* __restrict__ E, const int* __restrict__ tok, float* __restrict__ x, int d, int b,
                        int V) {
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < b * d; i += gridDim.x * blockDim.x) {
    const int bi = i / d, c = i - bi * d;
    const int t = tok[bi];
    x[i] = (t >= 0 && t < V) ? __bfloat162float(E[(size_t)t * d + c]) : __int_as_float(0x7fc00000);
  }
}

// xn = x / sqrt(mean(x^2) + eps) * g, one block per batch row
__global__ void rmsnorm_k(const float* __restrict__ x, const bf16* __restrict__ g, float* __restrict__ xn, int d,
                          float eps) {
  pdl_wait();
  __shared__ float red[32];
  const float* xr = x + (size_t)blockIdx.x * d;
  float s = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) s += xr[c] * xr[c];
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = 1.0f / sqrtf(v / (float)d + eps);
  }
  __syncthreads();
  const float r = red[0];
  for (int c = threadIdx.x; c < d; c += blockDim.x) xn[(size_t)blockIdx.x * d + c] = xr[c] * r * __bfloat162float(g[c]);
}

// out[bi][n] (+)= sum_k W[n][k] in[bi][k].  Rows n < n0 come from W0, n0 <= n < n1 from W1
// (row n - n0), the rest from W2 (row n - n1); every matrix has K columns.  Each warp takes
// R rows (more rows per warp share the activation loads at larger batches; fewer give more
// warps, and more loads in flight, at small ones); each lane 8 columns at a time with
// 16-byte loads.
template <int B, int R>
__global__ void gemv_k(const bf16* __restrict__ W0, const bf16* __restrict__ W1, const bf16* __restrict__ W2, int n0,
                       int n1, int N, int K, const float* __restrict__ in, float* __restrict__ out, int ld_out, int b,
                       int add) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * R;
  if (row0 >= N) return;
  const bf16* wr[R];
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const int n = min(row0 + j, N - 1);
    wr[j] = n < n0 ? W0 + (size_t)n * K : (n < n1 ? W1 + (size_t)(n - n0) * K : W2 + (size_t)(n - n1) * K);
  }
  float acc[R][B];
#pragma unroll
  for (int j = 0; j < R; ++j)
#pragma unroll
    for (int r = 0; r < B; ++r) acc[j][r] = 0.f;
#pragma unroll 4
  for (int k0 = lane * 8; k0 < K; k0 += 256) {
    float w[R][8];
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(wr[j] + k0));
      const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w[j][2 * e] = __uint_as_float(p[e] << 16);
        w[j][2 * e + 1] = __uint_as_float(p[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int r = 0; r < B; ++r) {
      if (r < b) {
        const float4 a0 = __ldg(reinterpret_cast<const float4*>(in + (size_t)r * K + k0));
        const float4 a1 = __ldg(reinterpret_cast<const float4*>(in + (size_t)r * K + k0 + 4));
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int j = 0; j < R; ++j)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[j][r] = fmaf(w[j][e], a[e], acc[j][r]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < R; ++j)
#pragma unroll
    for (int r = 0; r < B; ++r) acc[j][r] = warp_sum(acc[j][r]);
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int n = row0 + j;
      if (n >= N) break;
#pragma unroll
      for (int r = 0; r < B; ++r)
        if (r < b) {
          float* o = out + (size_t)r * ld_out + n;
          *o = add ? *o + acc[j][r] : acc[j][r];
        }
    }
}

// RoPE on the query and key heads of qkv [b][qdim + 2 kvdim] (rotate-half pairs, the fp32
// table), queries rotated in place, the new key and value appended to the cache in bf16.
// One block per (batch row, head of q|k|v), hd/2 threads.
__global__ void rope_append_k(float* __restrict__ qkv, const float2* __restrict__ rope, const int* __restrict__ pos,
                              const int* __restrict__ ptable, int mpps, bf16* __restrict__ kpool,
                              bf16* __restrict__ vpool, int layer, int num_pages, int nq, int nkv, int hd,
                              int max_ctx) {
  pdl_wait();
  const int heads = nq + 2 * nkv;
  const int bi = blockIdx.x / heads, hh = blockIdx.x - bi * heads;
  const int half = hd / 2, j = threadIdx.x;
  const int ldq = (nq + 2 * nkv) * hd;
  float* v = qkv + (size_t)bi * ldq + (size_t)hh * hd;
  const int p = pos[bi];
  if (p < 0 || p >= max_ctx || p / mk::kPage >= mpps) return;  // out of range: nothing written
  float x1 = v[j], x2 = v[j + half];
  if (hh < nq + nkv) {
    const float2 cs = rope[(size_t)p * half + j];
    const float o1 = x1 * cs.x - x2 * cs.y, o2 = x2 * cs.x + x1 * cs.y;
    x1 = o1;
    x2 = o2;
  }
  if (hh < nq) {
    v[j] = x1;
    v[j + half] = x2;
    return;
  }
  const int page = ptable[bi * mpps + p / mk::kPage];
  if (page < 0 || page >= num_pages) return;
  const int kvh = hh < nq + nkv ? hh - nq : hh - nq - nkv;
  bf16* dst = (hh < nq + nkv ? kpool : vpool) +
              ((((size_t)layer * num_pages + page) * nkv + kvh) * mk::kPage + p % mk::kPage) * hd;
  dst[j] = __float2bfloat16_rn(x1);
  dst[j + half] = __float2bfloat16_rn(x2);
}

// Split-K attention: one block per (batch row, kv head, chunk of kChunk keys), four warps
// taking the chunk's keys in turn, each with an online softmax per query head of the group;
// the warps merge in shared memory into one (O, m, l) partial per head.
template <int HD>
__global__ void attn_k(const float* __restrict__ qkv, const int* __restrict__ lens, const int* __restrict__ ptable,
                       int mpps, const bf16* __restrict__ kpool, const bf16* __restrict__ vpool, int layer, int num_pages,
                       int nq, int nkv, int nch, float* __restrict__ part) {
  pdl_wait();
  constexpr int PL = HD / 32;  // dims per lane
  const int g = nq / nkv;
  const int c = blockIdx.x % nch, pair = blockIdx.x / nch;
  const int bi = pair / nkv, kvh = pair - bi * nkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = min(lens[bi], mpps * mk::kPage);
  const int t0 = c * kChunk, t1 = min(n, t0 + kChunk);
  const size_t pst = (size_t)g * (HD + 2);
  float* pout = part + ((size_t)pair * nch + c) * pst;
  __shared__ float qs[8][HD];
  __shared__ float ws[4][8][HD + 2];
  const int ldq = (nq + 2 * nkv) * HD;
  for (int i = threadIdx.x; i < g * HD; i += blockDim.x)
    qs[i / HD][i % HD] = qkv[(size_t)bi * ldq + (size_t)(kvh * g) * HD + i] * rsqrtf((float)HD);
  __syncthreads();
  float m[8], l[8], o[8][PL];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < PL; ++e) o[h][e] = 0.f;
  }
  for (int t = t0 + warp; t < t1; t += 4) {
    const int page = ptable[bi * mpps + t / mk::kPage];
    if (page < 0 || page >= num_pages) continue;  // a missing page contributes nothing
    const size_t off = ((((size_t)layer * num_pages + page) * nkv + kvh) * mk::kPage + t % mk::kPage) * HD + lane * PL;
    float kv[PL], vv[PL];
    if constexpr (PL == 4) {
      const uint2 ku = *reinterpret_cast<const uint2*>(kpool + off), vu = *reinterpret_cast<const uint2*>(vpool + off);
      const uint32_t kw[2] = {ku.x, ku.y}, vw[2] = {vu.x, vu.y};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        kv[2 * e] = __uint_as_float(kw[e] << 16);
        kv[2 * e + 1] = __uint_as_float(kw[e] & 0xffff0000u);
        vv[2 * e] = __uint_as_float(vw[e] << 16);
        vv[2 * e + 1] = __uint_as_float(vw[e] & 0xffff0000u);
      }
    } else {
      const uint32_t ku = *reinterpret_cast<const uint32_t*>(kpool + off), vu = *reinterpret_cast<const uint32_t*>(vpool + off);
      kv[0] = __uint_as_float(ku << 16);
      kv[1] = __uint_as_float(ku & 0xffff0000u);
      vv[0] = __uint_as_float(vu << 16);
      vv[1] = __uint_as_float(vu & 0xffff0000u);
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h >= g) break;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < PL; ++e) s = fmaf(qs[h][lane * PL + e], kv[e], s);
      s = warp_sum(s);
      const float mn = fmaxf(m[h], s);
      const float corr = expf(m[h] - mn), pr = expf(s - mn);
      l[h] = l[h] * corr + pr;
#pragma unroll
      for (int e = 0; e < PL; ++e) o[h][e] = o[h][e] * corr + pr * vv[e];
      m[h] = mn;
    }
  }
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h < g) {
#pragma unroll
      for (int e = 0; e < PL; ++e) ws[warp][h][lane * PL + e] = o[h][e];
      if (lane == 0) {
        ws[warp][h][HD] = m[h];
        ws[warp][h][HD + 1] = l[h];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < g * HD; i += blockDim.x) {
    const int h = i / HD, dd = i % HD;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, ws[w][h][HD]);
    float A = 0.f, L = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float f = ws[w][h][HD] == -INFINITY ? 0.f : expf(ws[w][h][HD] - M);
      A += f * ws[w][h][dd];
      L += f * ws[w][h][HD + 1];
    }
    pout[h * (HD + 2) + dd] = A;
    if (dd == 0) {
      pout[h * (HD + 2) + HD] = M;
      pout[h * (HD + 2) + HD + 1] = L;
    }
  }
}

// The chunks' partials of one (batch row, kv head) merged: ao[bi][(kvh g + h) hd + d].
__global__ void combine_k(const float* __restrict__ part, const int* __restrict__ lens, int nq, int nkv, int hd, int nch,
                          float* __restrict__ ao) {
  pdl_wait();
  const int g = nq / nkv;
  const int pair = blockIdx.x, bi = pair / nkv, kvh = pair - bi * nkv;
  const int used = min((lens[bi] + kChunk - 1) / kChunk, nch);
  const size_t pst = (size_t)g * (hd + 2);
  const float* pp = part + (size_t)pair * nch * pst;
  for (int i = threadIdx.x; i < g * hd; i += blockDim.x) {
    const int h = i / hd, dd = i % hd;
    float M = -INFINITY;
    for (int c = 0; c < used; ++c) M = fmaxf(M, pp[c * pst + h * (hd + 2) + hd]);
    float A = 0.f, L = 0.f;
    for (int c = 0; c < used; ++c) {
      const float* q = pp + c * pst + h * (hd + 2);
      const float f = q[hd] == -INFINITY ? 0.f : expf(q[hd] - M);
      A += f * q[dd];
      L += f * q[hd + 1];
    }
    ao[(size_t)bi * nq * hd + (size_t)(kvh * g + h) * hd + dd] = A / L;
  }
}

// h[bi][j] = silu(gate) * up, from gu [b][2F] (gate rows, then up rows)
__global__ void swiglu_k(const float* __restrict__ gu, float* __restrict__ h, int F, int b) {
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < b * F; i += gridDim.x * blockDim.x) {
    const int bi = i / F, j = i - bi * F;
    const float gv = gu[(size_t)bi * 2 * F + j], uv = gu[(size_t)bi * 2 * F + F + j];
    h[i] = gv / (1.f + expf(-gv)) * uv;
  }
}

// greedy token per batch row: the lowest index of the maximum
__global__ void argmax_k(const float* __restrict__ logits, int V, int* __restrict__ out) {
  pdl_wait();
  __shared__ float bv[32];
  __shared__ int bix[32];
  const float* lr = logits + (size_t)blockIdx.x * V;
  float best = -INFINITY;
  int idx = 0x7fffffff;
  for (int i = threadIdx.x; i < V; i += blockDim.x) {
    const float v = lr[i];
    if (v > best || (v == best && i < idx)) { best = v; idx = i; }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (ov > best || (ov == best && oi < idx)) { best = ov; idx = oi; }
  }
  if ((threadIdx.x & 31) == 0) { bv[threadIdx.x >> 5] = best; bix[threadIdx.x >> 5] = idx; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
      if (bv[w] > best || (bv[w] == best && bix[w] < idx)) { best = bv[w]; idx = bix[w]; }
    out[blockIdx.x] = idx;
  }
}

// Launched in place of every kernel, with the same grid, in the empty mode: what is left
// of the step is the cost of its launches and kernel boundaries alone.
__global__ void noop_k() { pdl_wait(); }

}  // namespace kpo

// ---------------------------------------------------------------------------------------
// host side

struct mk_kpo_s {
  mk_model_cfg cfg{};
  std::vector<const bf16*> w[11];  // attn_norm wq wk wv wo mlp_norm w_gate w_up w_down (per layer)
  const bf16 *embed = nullptr, *final_norm = nullptr, *lm_head = nullptr;
  void* arena = nullptr;
  float *x, *xn, *qkv, *part, *ao, *gu, *h, *logits;
  int *tok, *pos, *lens, *argmax;
  float2* rope;
  int nch = 0;
  // the captured graph of one (batch, cache) combination
  cudaGraphExec_t graph = nullptr, empty = nullptr;
  int g_batch = 0, e_batch = 0;
  mk_kv_cache g_kv{}, e_kv{};
  std::string err;
};

static thread_local std::string kpo_err;

static int kpo_fail(mk_kpo_t k, int code, const std::string& msg) {
  (k ? k->err : kpo_err) = msg;
  return code;
}

#define KPO_CUDA(k, call)                                                                     \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess) return kpo_fail(k, MK_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

static bool g_noop = false;  // set while the empty mode's graph is captured (one thread at a time)

template <typename... KArgs, typename... Args>
static cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t s, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (g_noop) return cudaLaunchKernelEx(&cfg, kpo::noop_k);
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// One step's launches, in order.  `each` is called after every launch (the timed mode records
// an event there); a failed launch ends the sequence with its error.
template <class Each>
static cudaError_t enqueue_step(mk_kpo_t k, int b, const mk_kv_cache* kv, cudaStream_t s, bool pdl, Each each) {
  const mk_model_cfg& c = k->cfg;
  const int d = c.hidden, hd = c.head_dim, nq = c.n_heads, nkv = c.n_kv_heads, F = c.ffn, V = c.vocab;
  const int qdim = nq * hd, kvdim = nkv * hd, ldq = qdim + 2 * kvdim;
  const int wpb = 8;
  auto gemv = [&](const bf16* W0, const bf16* W1, const bf16* W2, int n0, int n1, int N, int K, const float* in,
                  float* out, int ld, int add) -> cudaError_t {
    const int R = b <= 2 ? 1 : (b <= 4 ? 2 : 4);
    const dim3 grid((N + wpb * R - 1) / (wpb * R)), block(32 * wpb);
    if (b == 1) return launch(kpo::gemv_k<1, 1>, grid, block, s, pdl, W0, W1, W2, n0, n1, N, K, in, out, ld, b, add);
    if (b == 2) return launch(kpo::gemv_k<2, 1>, grid, block, s, pdl, W0, W1, W2, n0, n1, N, K, in, out, ld, b, add);
    if (b <= 4) return launch(kpo::gemv_k<4, 2>, grid, block, s, pdl, W0, W1, W2, n0, n1, N, K, in, out, ld, b, add);
    return launch(kpo::gemv_k<8, 4>, grid, block, s, pdl, W0, W1, W2, n0, n1, N, K, in, out, ld, b, add);
  };
  cudaError_t e;
#define STEP(call)                    \
  do {                                \
    if ((e = (call)) != cudaSuccess) return e; \
    each();                           \
  } while (0)
  STEP(launch(kpo::embed_k, dim3((b * d + 255) / 256), dim3(256), s, pdl, k->embed, (const int*)k->tok, k->x, d, b, V));
  for (int l = 0; l < c.n_layers; ++l) {
    STEP(launch(kpo::rmsnorm_k, dim3(b), dim3(256), s, pdl, (const float*)k->x, k->w[0][l], k->xn, d, c.rms_eps));
    STEP(gemv(k->w[1][l], k->w[2][l], k->w[3][l], qdim, qdim + kvdim, ldq, d, k->xn, k->qkv, ldq, 0));
    STEP(launch(kpo::rope_append_k, dim3(b * (nq + 2 * nkv)), dim3(hd / 2), s, pdl, k->qkv, (const float2*)k->rope,
                (const int*)k->pos, kv->page_table, kv->max_pages_per_seq, (bf16*)kv->k_pool, (bf16*)kv->v_pool, l,
                kv->num_pages, nq, nkv, hd, c.max_ctx));
    if (hd == 64)
      STEP(launch(kpo::attn_k<64>, dim3(b * nkv * k->nch), dim3(128), s, pdl, (const float*)k->qkv, (const int*)k->lens,
                  kv->page_table, kv->max_pages_per_seq, (const bf16*)kv->k_pool, (const bf16*)kv->v_pool, l,
                  kv->num_pages, nq, nkv, k->nch, k->part));
    else
      STEP(launch(kpo::attn_k<128>, dim3(b * nkv * k->nch), dim3(128), s, pdl, (const float*)k->qkv,
                  (const int*)k->lens, kv->page_table, kv->max_pages_per_seq, (const bf16*)kv->k_pool,
                  (const bf16*)kv->v_pool, l, kv->num_pages, nq, nkv, k->nch, k->part));
    STEP(launch(kpo::combine_k, dim3(b * nkv), dim3(min(1024, (nq / nkv) * hd)), s, pdl, (const float*)k->part,
                (const int*)k->lens, nq, nkv, hd, k->nch, k->ao));
    STEP(gemv(k->w[4][l], k->w[4][l], k->w[4][l], d, d, d, qdim, k->ao, k->x, d, 1));
    STEP(launch(kpo::rmsnorm_k, dim3(b), dim3(256), s, pdl, (const float*)k->x, k->w[5][l], k->xn, d, c.rms_eps));
    STEP(gemv(k->w[6][l], k->w[7][l], k->w[7][l], F, 2 * F, 2 * F, d, k->xn, k->gu, 2 * F, 0));
    STEP(launch(kpo::swiglu_k, dim3((b * F + 255) / 256), dim3(256), s, pdl, (const float*)k->gu, k->h, F, b));
    STEP(gemv(k->w[8][l], k->w[8][l], k->w[8][l], d, d, d, F, k->h, k->x, d, 1));
  }
  STEP(launch(kpo::rmsnorm_k, dim3(b), dim3(256), s, pdl, (const float*)k->x, k->final_norm, k->xn, d, c.rms_eps));
  STEP(gemv(k->lm_head, k->lm_head, k->lm_head, V, V, V, d, k->xn, k->logits, V, 0));
  STEP(launch(kpo::argmax_k, dim3(b), dim3(256), s, pdl, (const float*)k->logits, V, k->argmax));
#undef STEP
  return cudaSuccess;
}

extern "C" {

MK_API int mk_kpo_create(const mk_model_cfg* cfg, const mk_weight_ptrs* w, mk_kpo_t* out) {
  if (!cfg || !w || !out) return kpo_fail(nullptr, MK_ERR_INVALID_ARG, "mk_kpo_create: null argument");
  std::string e;
  int rc = mk::check_cfg(*cfg, &e);
  if (rc) return kpo_fail(nullptr, rc, "mk_kpo_create: " + e);
  const mk_model_cfg& c = *cfg;
  if (c.max_batch > kpo::kMaxB || c.qk_norm || c.n_heads / c.n_kv_heads > 8)
    return kpo_fail(nullptr, MK_ERR_UNSUPPORTED_CFG,
                    "mk_kpo_create: the kernel-per-op step takes batches up to 8, no QK-norm, up to 8 query heads per kv head");
  if (!w->embed || !w->final_norm || !w->lm_head || !w->attn_norm || !w->wq || !w->wk || !w->wv || !w->wo ||
      !w->mlp_norm || !w->w_gate || !w->w_up || !w->w_down)
    return kpo_fail(nullptr, MK_ERR_INVALID_ARG, "mk_kpo_create: null weight pointer");
  mk_kpo_t k = new mk_kpo_s();
  k->cfg = c;
  const void* const* per[9] = {w->attn_norm, w->wq, w->wk, w->wv, w->wo, w->mlp_norm, w->w_gate, w->w_up, w->w_down};
  for (int a = 0; a < 9; ++a)
    for (int l = 0; l < c.n_layers; ++l) k->w[a].push_back((const bf16*)per[a][l]);
  k->embed = (const bf16*)w->embed;
  k->final_norm = (const bf16*)w->final_norm;
  k->lm_head = (const bf16*)w->lm_head;
  const int B = c.max_batch, d = c.hidden, hd = c.head_dim, nq = c.n_heads, nkv = c.n_kv_heads;
  const int qdim = nq * hd, ldq = qdim + 2 * nkv * hd;
  k->nch = (c.max_ctx + kpo::kChunk - 1) / kpo::kChunk;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~size_t(255); return o; };
  const size_t ox = take(4ull * B * d), oxn = take(4ull * B * d), oqkv = take(4ull * B * ldq);
  const size_t opart = take(4ull * B * nkv * k->nch * (nq / nkv) * (hd + 2)), oao = take(4ull * B * qdim);
  const size_t ogu = take(8ull * B * c.ffn), oh = take(4ull * B * c.ffn), ologits = take(4ull * B * c.vocab);
  const size_t otok = take(4ull * B), opos = take(4ull * B), olens = take(4ull * B), oam = take(4ull * B);
  const size_t orope = take(sizeof(float2) * (size_t)c.max_ctx * (hd / 2));
  cudaError_t ce = cudaMalloc(&k->arena, off);
  if (ce != cudaSuccess) {
    delete k;
    return kpo_fail(nullptr, MK_ERR_CUDA, std::string("mk_kpo_create: ") + cudaGetErrorString(ce));
  }
  unsigned char* A = (unsigned char*)k->arena;
  k->x = (float*)(A + ox); k->xn = (float*)(A + oxn); k->qkv = (float*)(A + oqkv); k->part = (float*)(A + opart);
  k->ao = (float*)(A + oao); k->gu = (float*)(A + ogu); k->h = (float*)(A + oh); k->logits = (float*)(A + ologits);
  k->tok = (int*)(A + otok); k->pos = (int*)(A + opos); k->lens = (int*)(A + olens); k->argmax = (int*)(A + oam);
  k->rope = (float2*)(A + orope);
  ce = mk::launch_rope_table(k->rope, c.max_ctx, hd, mk_rope_freq(c), 0);
  if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
  if (ce != cudaSuccess) {
    cudaFree(k->arena);
    delete k;
    return kpo_fail(nullptr, MK_ERR_CUDA, std::string("mk_kpo_create: ") + cudaGetErrorString(ce));
  }
  *out = k;
  return MK_OK;
}

MK_API int mk_kpo_step(mk_kpo_t k, const int32_t* token_ids, const int32_t* positions, const int32_t* seq_lens,
                       int32_t batch, const mk_kv_cache* kv, float* logits_out, int32_t* argmax_out, int32_t mode,
                       float* busy_ms, mk_stream_t stream) {
  if (!k) return kpo_fail(nullptr, MK_ERR_INVALID_ARG, "mk_kpo_step: null handle");
  if (!token_ids || !positions || !seq_lens || !kv || !logits_out)
    return kpo_fail(k, MK_ERR_INVALID_ARG, "mk_kpo_step: null argument");
  if (batch < 1 || batch > k->cfg.max_batch) return kpo_fail(k, MK_ERR_INVALID_ARG, "mk_kpo_step: batch out of range");
  if (!kv->k_pool || !kv->v_pool || !kv->page_table || kv->num_pages < 1 || kv->max_pages_per_seq < 1)
    return kpo_fail(k, MK_ERR_INVALID_ARG, "mk_kpo_step: bad kv cache description");
  if (mode < MK_KPO_GRAPH || mode > MK_KPO_EMPTY) return kpo_fail(k, MK_ERR_INVALID_ARG, "mk_kpo_step: unknown mode");
  const cudaStream_t s = (cudaStream_t)stream;
  const size_t ib = sizeof(int32_t) * batch;
  KPO_CUDA(k, cudaMemcpyAsync(k->tok, token_ids, ib, cudaMemcpyDeviceToDevice, s));
  KPO_CUDA(k, cudaMemcpyAsync(k->pos, positions, ib, cudaMemcpyDeviceToDevice, s));
  KPO_CUDA(k, cudaMemcpyAsync(k->lens, seq_lens, ib, cudaMemcpyDeviceToDevice, s));
  if (mode == MK_KPO_GRAPH || mode == MK_KPO_EMPTY) {
    const bool noop = mode == MK_KPO_EMPTY;
    cudaGraphExec_t& ge = noop ? k->empty : k->graph;
    int& gb = noop ? k->e_batch : k->g_batch;
    mk_kv_cache& gkv = noop ? k->e_kv : k->g_kv;
    if (!(ge && gb == batch && std::memcmp(&gkv, kv, sizeof(*kv)) == 0)) {
      if (ge) cudaGraphExecDestroy(ge);
      ge = nullptr;
      cudaStream_t cs;
      KPO_CUDA(k, cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
      cudaGraph_t g = nullptr;
      cudaError_t e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
      if (e == cudaSuccess) {
        g_noop = noop;
        const cudaError_t e1 = enqueue_step(k, batch, kv, cs, true, [] {});
        g_noop = false;
        e = cudaStreamEndCapture(cs, &g);
        if (e1 != cudaSuccess) e = e1;
      }
      if (e == cudaSuccess) e = cudaGraphInstantiate(&ge, g, 0);
      if (g) cudaGraphDestroy(g);
      cudaStreamDestroy(cs);
      if (e != cudaSuccess) {
        ge = nullptr;
        return kpo_fail(k, MK_ERR_CUDA, std::string("mk_kpo_step: graph capture: ") + cudaGetErrorString(e));
      }
      gb = batch;
      gkv = *kv;
    }
    KPO_CUDA(k, cudaGraphLaunch(ge, s));
    if (noop) return MK_OK;  // no results to copy
  } else if (mode == MK_KPO_STREAM) {
    KPO_CUDA(k, enqueue_step(k, batch, kv, s, true, [] {}));
  } else {
    // every kernel between two events, no launch overlap: the sum is the device time the
    // kernels themselves take
    std::vector<cudaEvent_t> ev;
    cudaEvent_t e0;
    KPO_CUDA(k, cudaEventCreate(&e0));
    ev.push_back(e0);
    KPO_CUDA(k, cudaEventRecord(e0, s));
    cudaError_t err = cudaSuccess;
    const cudaError_t e = enqueue_step(k, batch, kv, s, false, [&] {
      cudaEvent_t x;
      if (err == cudaSuccess) err = cudaEventCreate(&x);
      if (err == cudaSuccess) {
        ev.push_back(x);
        err = cudaEventRecord(x, s);
      }
    });
    if (e != cudaSuccess) err = e;
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    float total = 0.f;
    for (size_t i = 1; err == cudaSuccess && i < ev.size(); ++i) {
      float ms = 0.f;
      err = cudaEventElapsedTime(&ms, ev[i - 1], ev[i]);
      total += ms;
    }
    for (cudaEvent_t x : ev) cudaEventDestroy(x);
    if (err != cudaSuccess) return kpo_fail(k, MK_ERR_CUDA, std::string("mk_kpo_step: ") + cudaGetErrorString(err));
    if (busy_ms) *busy_ms = total;
  }
  KPO_CUDA(k, cudaMemcpyAsync(logits_out, k->logits, sizeof(float) * (size_t)batch * k->cfg.vocab,
                              cudaMemcpyDeviceToDevice, s));
  if (argmax_out) KPO_CUDA(k, cudaMemcpyAsync(argmax_out, k->argmax, ib, cudaMemcpyDeviceToDevice, s));
  return MK_OK;
}

MK_API int mk_kpo_launches_per_step(mk_kpo_t k) { return k ? 10 * k->cfg.n_layers + 4 : MK_ERR_INVALID_ARG; }

MK_API int mk_kpo_destroy(mk_kpo_t k) {
  if (!k) return MK_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  if (k->graph) cudaGraphExecDestroy(k->graph);
  if (k->empty) cudaGraphExecDestroy(k->empty);
  if (k->arena) cudaFree(k->arena);
  delete k;
  return MK_OK;
}

MK_API const char* mk_kpo_last_error(mk_kpo_t k) { return k ? k->err.c_str() : kpo_err.c_str(); }

}  // extern "C"
