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
constexpr int kProducerWarp = kConsumerWarps;           // weight and KV copies
constexpr int kOperandWarp = kConsumerWarps + 1;        // GEMV operand copies
constexpr int kSignalWarp = kConsumerWarps + 2;         // releases finished tasks' counters
constexpr int kThreads = (kConsumerWarps + 3) * 32;
constexpr int kSigRing = 4;                             // finished tasks the consumers may run ahead of their release
constexpr int kSlotBytes = 50 * 1024;                   // one pool stage: weights + their operands, or KV pages
constexpr int kNumSlots = 4;                            // pool depth (200 KB; 4 x 50 KB measured fastest)
constexpr int kMaxBatch = 16;
constexpr int kFmaRows = 2;                             // batches up to this size run the GEMVs on fp32 FMA
constexpr int kTriRows = 4;                             // batches up to this size split activations in three bf16 parts
constexpr int kMaxBlocks = 8;                           // 8-row blocks per GEMV task (64 rows)
constexpr int kPage = 16;                               // tokens per KV page
constexpr int kMaxChunksPerSeq = 32;                    // split-K chunks per (sequence, kv head)
constexpr int kMaxTopK = 256;                           // largest k of top-k sampling
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

// A GEMV task group may be cut along K into up to kMaxPieces pieces; split tag = id << 4 |
// piece << 2 | (pieces - 1), id = the group's K-piece partial slot.
constexpr uint16_t kNoSplit = 0xFFFF;
constexpr int kMaxPieces = 4;
MK_HD uint16_t split_tag(int id, int piece, int pieces) { return (uint16_t)((id << 4) | (piece << 2) | (pieces - 1)); }
MK_HD int split_id(uint16_t s) { return s >> 4; }
MK_HD int split_piece(uint16_t s) { return (s >> 2) & 3; }
MK_HD int split_pieces(uint16_t s) { return (s & 3) + 1; }

struct TaskDesc {          // 32 bytes, read by every thread of the CTA
  uint8_t op;
  uint8_t nunits;          // work units covered: [u0, u0 + nunits)
  uint16_t layer;
  uint32_t u0;
  uint16_t task_idx;       // index of this task within its phase (partial-result slot)
  uint16_t kc;             // K columns per pool stage (GEMV tasks)
  uint16_t wait_ctr;       // counter to wait on before reading activations (kNoCounter: none)
  uint16_t sig_ctr;        // counter this task adds one to when it is done
  uint32_t wait_count;     // signals per step the wait needs: target = wait_count * epoch
  uint16_t k0, k1;         // GEMV: the 64-column chunks [k0, k1) of K the task covers
  uint16_t split;          // kNoSplit, or split_tag(id, piece, pieces) for a K piece of a task group
  uint16_t slot0;          // per-task partial slot the task group's result goes to (piece 0's task_idx)
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

// fp32 operand rows a stage carries for a batch of b <= kFmaRows rows (1 or 2).
MK_HD int fma_rows(int b) { return b == 1 ? 1 : kFmaRows; }

// Operand bytes per K column of one stage for a batch of up to max_batch rows: bf16 hi and
// lo parts of every 8-row batch tile (16 bytes each per column), or, when every batch the
// handle takes runs on the fp32 path (max_batch <= kFmaRows), 4 bytes per fp32 row.  A
// batch-1 handle thus streams 384 weight columns of a 64-row task per 50 KB stage, not 320.
MK_HD int operand_col_bytes(int max_batch) {
  return max_batch <= kFmaRows ? 4 * fma_rows(max_batch) : 32 * ((max_batch + 7) / 8);
}

// K columns per pool stage of a GEMV task with `blocks` 8-row blocks: the largest multiple of
// 64 whose weights (blocks * 8 rows) and operands fit one slot, at most K rounded up to 64.
MK_HD int stage_cols(int blocks, int K, int max_batch) {
  const int per_col = blocks * 8 * 2 + operand_col_bytes(max_batch);
  int kc = (kSlotBytes / per_col) / kBoxCols * kBoxCols;
  if (kc < kBoxCols) kc = kBoxCols;
  const int kp = round_up(K, kBoxCols);
  return kp <= kc ? kp : kc;
}

// Operand layouts in global memory, written by the producing epilogues and copied per stage
// by tiled TMA boxes into the slot, where the consuming lanes read them.  A 64-column chunk c
// holds two 32-column k blocks kb = 2c + h: block h takes the 16-byte column groups 2tq + h
// (tq = 0..3) of the chunk, the groups lane (g, tq) reads from its weight rows.
//   bf16 tiles: per batch tile mt (rows 8mt..8mt+7) and part (0 hi, 1 lo), block kb is 512
//   contiguous bytes: 32 pieces of 16 bytes, piece 4 * row + tq = the 8 columns of group
//   2tq + h of batch row `row` - lane (g, tq) reads piece `lane`;
//   fp32 batch rows 0..kFmaRows-1, each ld values: block kb is 128 bytes, piece tq = the 8
//   values of group 2tq + h.
MK_HD int opnd_block(int k) { return ((k >> 6) << 1) | ((k >> 3) & 1); }
MK_HD size_t opnd_tile_index(int mt, int part, int k, int row, int ld) {
  return ((((size_t)(mt * 2 + part) * (ld / 32) + opnd_block(k)) * 32 + row * 4 + ((k >> 4) & 3)) * 8 + (k & 7));
}
MK_HD size_t opnd_row0_index(int k) { return ((size_t)opnd_block(k) * 4 + ((k >> 4) & 3)) * 8 + (k & 7); }

// Index of the TMA descriptor of weight matrix `mat` (0 wq .. 6 w_down) of a layer for
// boxes of 8*n rows; the LM head's maps follow the layers' (mat 0 of layer L).
MK_HD int tmap_index(int layer, int mat, int n) { return (layer * kNumMats + mat) * kMaxBlocks + (n - 1); }

MK_HD int num_tmaps(int n_layers) { return (n_layers + 1) * kNumMats * kMaxBlocks; }

// Operand tensor maps, after the weight maps: per operand kind (0 normed x, 1 attention
// output, 2 SwiGLU output), 2 * tiles bf16 maps (tile mt, part) then the map of the fp32 rows.
constexpr int kMaxTiles = (kMaxBatch + 7) / 8;
constexpr int kOpMapsPerKind = 2 * kMaxTiles + 1;
MK_HD int opmap_index(int n_layers, int kind, int q) { return num_tmaps(n_layers) + kind * kOpMapsPerKind + q; }
MK_HD int num_all_tmaps(int n_layers) { return num_tmaps(n_layers) + 3 * kOpMapsPerKind; }

// Tokens per attention stage: K rows then V rows of the same tokens, 32 KB (head_dim 64) or
// 48 KB (head_dim 128: six 16-token warp groups on one stage, most of a 50 KB slot).
MK_HD int attn_stage_tokens(int head_dim) { return head_dim == 64 ? 128 : 96; }

}  // namespace mk
