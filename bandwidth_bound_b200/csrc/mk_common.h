// Shared host/device definitions of the decode megakernel: the task descriptor
// that per-SM instruction streams are made of, the work units each task type
// covers, the dependency-counter numbering and the stage geometry.
//
// The structure follows "ForgeMegakernel: A General Framework for Efficient
// Auto-Regressive Model Decode Megakernels" (§4.1 "The universal knowledge base
// and the milestones": a fine-grained instruction stream per SM, dependency
// counters instead of grid-wide barriers, a shared-memory buffer pool) and the
// "Inside the megakernel serving engine" digest (one persistent thread block per
// SM, task descriptors, counter-based barriers in global memory, weights streamed
// into shared memory before activation dependencies are met).
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define MK_HD __host__ __device__ __forceinline__
#else
#define MK_HD inline
#endif

namespace mk {

// ---- launch geometry -------------------------------------------------------------------
constexpr int kConsumerWarps = 8;                       // compute warps per CTA
constexpr int kThreads = (kConsumerWarps + 1) * 32;     // + one producer (TMA) warp
constexpr int kSlotBytes = 32 * 1024;                   // one pool stage: weights or KV pages (1024-byte aligned)
constexpr int kNumSlots = 5;                            // pool depth (160 KB)
constexpr int kRingBytes = 4 * 1024;                    // per consumer warp: GEMV operands of its next k blocks
constexpr int kMaxBatch = 16;
constexpr int kMaxBlocks = 8;                           // 8-row blocks per GEMV task (64 rows)
constexpr int kPage = 16;                               // tokens per KV page
constexpr int kMaxChunksPerSeq = 32;                    // split-K chunks per (sequence, kv head)
constexpr int kRedBytes = kConsumerWarps * kMaxBlocks * 8 * 8 * 4;   // 16 KB: one 8-row batch tile at a time
constexpr int kNoCounter = 0xFFFF;
constexpr int kBoxCols = 64;                            // weight columns per TMA box (128 bytes, 128B swizzle)
constexpr int kNumMats = 7;                             // wq wk wv wo w_gate w_up w_down

// ---- task descriptors -------------------------------------------------------------------
enum Op : uint8_t {
  OP_EMBED = 1,   // x = E[token]; units: 8 hidden columns
  OP_QKV = 2,     // q,k,v = W xn, RoPE, KV append; unit: rows (8m..8m+7) and (hd/2+8m..) of one head
  OP_ATTN = 3,    // split-K flash-decode slot; u0 = global slot index
  OP_OPROJ = 4,   // x += Wo attn; unit: 8 rows of Wo
  OP_GATEUP = 5,  // h = silu(Wg xn) * (Wu xn); unit: rows 8u..8u+7 of Wg and of Wu
  OP_DOWN = 6,    // x += Wd h; unit: 8 rows of Wd
  OP_LMHEAD = 7,  // logits = Wlm xn; unit: 8 rows of the LM head
};

struct TaskDesc {          // 24 bytes, read by every thread of the CTA
  uint8_t op;
  uint8_t nunits;          // work units covered: [u0, u0 + nunits)
  uint16_t layer;
  uint32_t u0;
  uint16_t task_idx;       // index of this task within its phase (partial-result slot)
  uint16_t kc;             // K columns per pool stage (GEMV tasks)
  uint16_t wait_ctr;       // counter to wait on before reading activations (kNoCounter: none)
  uint16_t sig_ctr;        // counter this task adds one to when it is done
  uint32_t wait_count;     // signals per step the wait needs: target = wait_count * epoch
};

// ---- counters ---------------------------------------------------------------------------
// 0: embed; 1 + 5*l + k for layer l, k = 0 qkv, 1 attn, 2 oproj, 3 gateup, 4 down; 1 + 5*L: lm head
MK_HD int ctr_embed() { return 0; }
MK_HD int ctr_layer(int l, int k) { return 1 + 5 * l + k; }
MK_HD int ctr_lm(int L) { return 1 + 5 * L; }
MK_HD int num_counters(int L) { return 2 + 5 * L; }

// Partial sums of squares of the residual stream, one instance per residual writer:
// 0 embed, 1 + 2l oproj of layer l, 2 + 2l down of layer l.
MK_HD int ssq_inst_embed() { return 0; }
MK_HD int ssq_inst_oproj(int l) { return 1 + 2 * l; }
MK_HD int ssq_inst_down(int l) { return 2 + 2 * l; }
MK_HD int num_ssq_inst(int L) { return 1 + 2 * L; }

// ---- units ------------------------------------------------------------------------------
MK_HD int rows_per_unit(int op) { return (op == OP_QKV || op == OP_GATEUP) ? 16 : 8; }
MK_HD int max_units(int op) { return (op == OP_QKV || op == OP_GATEUP) ? kMaxBlocks / 2 : kMaxBlocks; }

MK_HD uint32_t ceil_div(uint32_t a, uint32_t b) { return (a + b - 1) / b; }
MK_HD int round_up(int a, int b) { return (a + b - 1) / b * b; }

// K columns per pool stage of a GEMV task with `blocks` 8-row blocks: the weights fit a
// slot and every consumer warp gets whole 32-column blocks (1, 2 or 4 of them).
MK_HD int stage_cols(int blocks, int K, int max_batch) {
  (void)max_batch;
  const int kc = blocks >= 5 ? 256 : (blocks >= 3 ? 512 : 1024);
  const int kp = round_up(K, kBoxCols);
  return kp <= kc ? kp : kc;
}

// Operand tile layout in global memory (written by the producing epilogues, read by the
// consuming GEMV's lanes): for batch tile mt (rows 8mt..8mt+7) and part (0 hi, 1 lo),
// groups of 8 columns; group kg holds 8 rows of 16 bytes (row g in slot g ^ (2 * ((kg >> 1)
// & 3)), a permutation that keeps every 128-byte group whole for the reading warp).
MK_HD size_t operand_index(int mt, int part, int kg, int g, int e, int ld) {
  return ((((size_t)(mt * 2 + part) * (ld / 8) + kg) * 8 + (g ^ (2 * ((kg >> 1) & 3)))) * 8 + e);
}

// Index of the TMA descriptor of weight matrix `mat` (0 wq .. 6 w_down) of a layer for
// boxes of 8*n rows; the LM head's maps follow the layers' (mat 0 of layer L).
MK_HD int tmap_index(int layer, int mat, int n) { return (layer * kNumMats + mat) * kMaxBlocks + (n - 1); }

MK_HD int num_tmaps(int n_layers) { return (n_layers + 1) * kNumMats * kMaxBlocks; }

// Tokens per attention stage: K rows then V rows of the same tokens, 32 KB total.
MK_HD int attn_stage_tokens(int head_dim) { return head_dim == 64 ? 128 : 64; }

}  // namespace mk
