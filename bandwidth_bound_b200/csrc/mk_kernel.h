// Kernel parameters of the decode megakernel (internal header).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mk_common.h"

namespace mk {

struct LayerW {
  const __nv_bfloat16 *attn_norm, *wq, *wk, *wv, *wo, *mlp_norm, *wg, *wu, *wd;
};

struct KParams {
  // model shape
  int L, d, nq, nkv, hd, F, V, g, qdim, max_b, max_ctx;
  float eps;
  const LayerW* layers;  // device [L]
  const __nv_bfloat16 *embed, *final_norm, *lm_head;
  // schedule
  const TaskDesc* tasks;
  const uint32_t* task_off;  // [num_sms + 1]
  int num_sms, n_slots, n_lm_tasks;
  // handle-owned device state
  float *x, *q, *attn, *hbuf, *ssq, *part;
  int ssq_stride;            // floats per ssq instance
  float2* lmpart;            // [n_lm_tasks][max_b] (value, index bits)
  uint32_t *ctr, *cmb, *ctl; // counters, split-K combine counters, {abort, status}
  int* host_status;          // mapped host word
  const float2* rope;        // [max_ctx][hd/2] (cos, sin)
  // this step
  const int *tok, *pos, *lens;
  int b;
  __nv_bfloat16 *kpool, *vpool;
  const int* ptable;
  int num_pages, mpps;
  float* logits;
  int* argmax;
  float* dbg;
  uint32_t epoch;
  unsigned long long timeout_ns;
};

size_t kernel_smem_bytes();
cudaError_t launch_decode(const KParams& p, cudaStream_t s);
cudaError_t launch_rope_table(float2* table, int max_ctx, int hd, double theta, cudaStream_t s);
cudaError_t kernel_attributes(int* regs, int* local_bytes, int* max_threads);

}  // namespace mk
