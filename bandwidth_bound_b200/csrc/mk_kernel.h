// Kernel parameters of the decode megakernel (internal header).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mk_common.h"

namespace mk {

struct LayerW {
  const __nv_bfloat16 *attn_norm, *wq, *wk, *wv, *wo, *mlp_norm, *wg, *wu, *wd;
  const __nv_bfloat16 *q_norm, *k_norm;  // QK-norm gains [hd] (null without QK-norm)
};

struct alignas(64) TmaDesc {  // the driver's opaque 128-byte TMA descriptor (CUtensorMap)
  unsigned long long v[16];
};

struct KParams {
  // this step's KV pools as tiled maps (16-token page boxes, 128-byte swizzle), encoded by
  // the host when the pools change
  TmaDesc kmap, vmap;
  // model shape
  int L, d, nq, nkv, hd, F, V, g, qdim, max_b, max_ctx;
  float eps;
  const LayerW* layers;  // device [L]
  const __nv_bfloat16 *embed, *final_norm, *lm_head;
  // schedule
  const TaskDesc* tasks;
  const uint32_t* task_off;  // [num_sms + 1]
  int num_sms, n_slots, n_lm_tasks;
  const void* tmaps;          // CUtensorMap array: weights (tmap_index) then the LM head
  // handle-owned device state
  float *x, *q, *ssq;
  float* part;               // split-K partials [max_b * nkv][kMaxChunksPerSeq][g][hd + 2]
  // GEMV operands, written once by the producing phase: bf16 hi/lo tiles in the layout of
  // operand_index (all batch rows) and fp32 (batch rows below kFmaRows, for the FMA path).
  // ax: x * gain of the next RMSNorm (input of qkv / gate-up / lm head), aa: attention output,
  // ah: SwiGLU output; ld = K rounded up to 64, padding zero
  __nv_bfloat16 *ax_t, *aa_t, *ah_t;
  float *ax_f, *aa_f, *ah_f;
  int ld_x, ld_a, ld_h;
  int ssq_stride;            // floats per ssq instance
  float2* lmpart;            // [n_lm_tasks][max_b] (value, index bits)
  int2* lmrows;              // [n_lm_tasks] (first vocabulary row, rows) of the task whose maxima lmpart holds
  float* spart;              // K-piece partial sums [split id][kMaxPieces][64 rows][max_b]
  uint32_t* scnt;            // K-piece arrival counters [split id]
  int n_split;               // split ids (entries of scnt)
  uint32_t *ctr, *cmb, *ctl; // counters, split-K combine counters, {abort, status}
  int* host_status;          // mapped host word
  const float2* rope;        // [max_ctx][hd/2] (cos, sin)
  // QK-norm: per (batch row, q or k head) partial sums of squares of the raw head vector,
  // one slot per 16-row QKV unit of the head [max_b][nq + nkv][hd / 16]; the new keys
  // rotated but not yet normalised [max_b][nkv][hd] (the attention task holding the new
  // position normalises and stores them)
  int qk_norm;
  float *qkss, *knew;
  // this step
  const int *tok, *pos, *lens;  // lens may be null: pos + 1
  int b;
  int step_add;                 // added to every position (and length): step index of a multi-step run
  const int* group_first;       // multi-token step: first row of each row's sequence (null: every row its own)
  __nv_bfloat16 *kpool, *vpool;
  const int* ptable;
  int num_pages, mpps;
  float* logits;
  int* argmax;                 // the step's next token per sequence: greedy, or drawn from the top_k
  int top_k;                   // <= 1: greedy; 2..kMaxTopK: sample among the top_k logits
  float temperature;           // > 0 (sampling only)
  const float* uniforms;       // [b] in [0, 1): this step's draw per sequence (sampling only)
  float* dbg;
  uint32_t epoch;
  unsigned long long timeout_ns;
  unsigned long long* trace;  // optional [n_tasks][4] records (see mk_set_trace)
};

size_t kernel_smem_bytes();
cudaError_t launch_decode(const KParams& p, cudaStream_t s);
struct RopeFreq {
  double inv_freq[64];  // per rotation pair j < hd / 2
};
cudaError_t launch_rope_table(float2* table, int max_ctx, int hd, const RopeFreq& f, cudaStream_t s);

cudaError_t kernel_attributes(int* regs, int* local_bytes, int* max_threads);

}  // namespace mk

// RoPE inverse frequencies of a model cfg (the scaling rule of mk_model_cfg), in double.
struct mk_model_cfg;
mk::RopeFreq mk_rope_freq(const mk_model_cfg& c);
