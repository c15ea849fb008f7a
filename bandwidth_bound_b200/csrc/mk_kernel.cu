// The decode megakernel for B200 (sm_100a): one persistent CTA per SM.
//
// Structure (from "ForgeMegakernel: A General Framework for Efficient
// Auto-Regressive Model Decode Megakernels", §2.1, §2.3 and §4.1, and the
// "Inside the megakernel serving engine" digest):
//   * the whole decode step is one launch; each CTA walks its own host-built
//     stream of task descriptors;
//   * tasks wait on dependency counters in global memory (acquire loads) and
//     signal them (release read-modify-writes) instead of grid-wide barriers;
//   * a shared-memory pool of stage slots is filled ahead of the compute: one
//     producer warp streams every weight tile and KV page of the CTA's whole stream
//     (they do not depend on this step's activations), one operand warp adds each
//     GEMV stage's activation slice once the task's dependency is met, and eight
//     consumer warps compute from the slots.
// B200 choices: every copy is a tiled TMA box (cp.async.bulk.tensor, no multicast)
// with completion on mbarriers; evict-first L2 policy for streamed bytes; fp32
// accumulation; CUDA-core FMA GEMV at batch 1; mma.sync bf16 tensor cores with hi/lo
// split activations at batch >= 2; split-K flash-decode attention with both products on
// tensor cores (ldmatrix fragments from 128-byte-swizzled page boxes).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mk_kernel.h"

// Cycle accounting inside a task (per-stage compute and slot waits, reduce and epilogue
// time) for the per-task timeline.  Off by default: the stamps sit in the hot loops and cost
// ~2-3 % of the step.  Timestamps per task (start, dependency met, end) are always recorded
// when a timeline buffer is set.
#ifndef MK_TRACE_DETAIL
#define MK_TRACE_DETAIL 0
#endif

namespace mk {

typedef __nv_bfloat16 bf16;
typedef TmaDesc CUtensorMapLike;

// ---------------------------------------------------------------------------------------
// shared memory

struct Smem {
  alignas(1024) uint8_t pool[kNumSlots][kSlotBytes];  // per slot: weight boxes + operands, or KV pages, of one stage
  alignas(16) float red[kRedBytes / 4];                 // GEMV cross-warp partials / attention merge
  alignas(16) float ep[kMaxBlocks * 8][kMaxBatch];       // per-task results [row][batch]
  float mw[kConsumerWarps][8], lw[kConsumerWarps][8];    // attention merge state per warp
  float inv_rms[kMaxBatch];
  alignas(8) uint64_t wfull[kNumSlots];                  // the stage landed: weights or KV (producer) and
                                                         // operands (operand warp), two arrivals
  alignas(8) uint64_t empty[kNumSlots];                  // all consumer warps done with the stage
  alignas(8) uint64_t sigfull[kSigRing];                 // consumer warps: task done, its writes ordered before
  alignas(8) uint64_t sigempty[kSigRing];                // signal warp: that task's counter released
  int sigab[kSigRing];                                   // the consumers gave up on that task (no release)
  int lm_last;                                           // this CTA released the step's last LM-head task
  int attn_R, bad, flag, flag2;  // attn_R: tokens per attention range on the pair line (this step), 0: pair-aligned
  int attn_n[kMaxBatch];         // pair-aligned: ranges per (sequence i, kv head) pair
  int attn_Ri[kMaxBatch];        // pair-aligned: tokens per range of sequence i (a multiple of 16)
  int attn_u0[kMaxBatch + 1];    // pair-aligned: first range of sequence i
  int in_tok[kMaxBatch];         // this step's token, position and keys attended per sequence,
  int in_pos[kMaxBatch];         // read once from the step's inputs (positions offset by the
  int in_len[kMaxBatch];         // step's index in a multi-step run)
  int in_grow0[kMaxBatch];       // multi-token step: first batch row of the row's sequence
  int in_fresh[kMaxBatch];       // first position written by this step in the row's sequence
  unsigned long long wait_cyc;  // tracing: SM cycles warp 0 spent waiting for pool slots in the current task
  unsigned long long tm[3];     // tracing: compute, reduce, epilogue SM cycles of the current task (warp 0)
};

size_t kernel_smem_bytes() { return sizeof(Smem); }

// ---------------------------------------------------------------------------------------
// PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of an mbarrier phase (try_wait may suspend the caller for a while).
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Tiled TMA loads of a box of a weight matrix (128-byte swizzle), completion on an mbarrier.
__device__ __forceinline__ void tma_2d(void* dst, const void* map, int c0, int c1, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_3d(void* dst, const void* map, int c0, int c1, int c2, uint64_t* bar,
                                       uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t atom_add_acqrel(uint32_t* p, uint32_t v) {
  uint32_t o;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(o) : "l"(p), "r"(v) : "memory");
  return o;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void cbar() {  // the consumer warps only
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---------------------------------------------------------------------------------------
// errors, waits

__device__ __noinline__ void raise_error(const KParams& p, int code) {
  if (atomicCAS(reinterpret_cast<int*>(&p.ctl[1]), 0, code) == 0) {
    *reinterpret_cast<volatile int*>(p.host_status) = code;
    __threadfence_system();
  }
  atomicExch(&p.ctl[0], 1u);
}

__device__ __forceinline__ bool aborted(const KParams& p) { return ld_relaxed(&p.ctl[0]) != 0; }

// Wait until the mbarrier phase of the given parity completes.  Bounded: gives up
// (returning false) when the abort flag is set or the time limit passes.
__device__ bool mbar_wait(const KParams& p, uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 15) == 0) {
      if (aborted(p)) return false;
      if (gtimer() - t0 > p.timeout_ns) {
        raise_error(p, -5 /* MK_ERR_DEVICE_TIMEOUT */);
        return false;
      }
    }
  }
}

// Non-blocking test that stage `st` has landed (weights and operands complete one barrier);
// issued ahead of a stage's compute, its ~200-cycle latency overlaps that.
__device__ __forceinline__ uint32_t stage_landed(Smem& sm, uint32_t st) {
  const int slot = st % kNumSlots;
  const uint32_t par = (st / kNumSlots) & 1;
  return mbar_test(&sm.wfull[slot], par) ? 1u : 0u;
}

// Warp-wide wait, taken by whole warps (copy warps, consumer stage waits, signal warp): every
// lane tests the barrier (one shared-memory request) and a vote makes the answer uniform, so
// no lane waits alone and then broadcasts; the polling loop checks the abort flag and the
// time limit (decided by vote too).  Inlined, like every function on the step's paths but
// the error report and the sampler: a call costs a warp its live registers' spills and
// refills after the wait (out of line, the waits and the QK-norm epilogue cost 1.5 % at b8).
__device__ __forceinline__ bool mbar_wait_all_slow(const KParams& p, uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = gtimer();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
    if ((it & 15) == 0) {
      const bool late = gtimer() - t0 > p.timeout_ns;
      if (__any_sync(0xffffffffu, aborted(p) || late)) {
        if ((threadIdx.x & 31) == 0 && late && !aborted(p)) raise_error(p, -5 /* MK_ERR_DEVICE_TIMEOUT */);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait_all(const KParams& p, uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_try(bar, parity)) || mbar_wait_all_slow(p, bar, parity);
}

// Wait until counter c has received count*epoch signals (wrap-around safe).
__device__ bool wait_counter(const KParams& p, int c, uint32_t count) {
  const uint32_t target = count * p.epoch;
  const uint32_t* ptr = p.ctr + c;
  if ((int32_t)(ld_acquire(ptr) - target) >= 0) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if ((int32_t)(ld_acquire(ptr) - target) >= 0) return true;
    if ((it & 15) == 0) {
      if (aborted(p)) return false;
      if (gtimer() - t0 > p.timeout_ns) {
        raise_error(p, -5);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_counter_all_slow(const KParams& p, const uint32_t* ptr, uint32_t target) {
  const uint64_t t0 = gtimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (__all_sync(0xffffffffu, (int32_t)(ld_acquire(ptr) - target) >= 0)) return true;
    if ((it & 15) == 0) {
      const bool late = gtimer() - t0 > p.timeout_ns;
      if (__any_sync(0xffffffffu, aborted(p) || late)) {
        if ((threadIdx.x & 31) == 0 && late && !aborted(p)) raise_error(p, -5);
        return false;
      }
    }
  }
}
// Warp-wide counter wait: every lane loads the counter (one request per warp), a vote makes
// the answer uniform.
__device__ __forceinline__ bool wait_counter_all(const KParams& p, int c, uint32_t count) {
  const uint32_t target = count * p.epoch;
  const uint32_t* ptr = p.ctr + c;
  return __all_sync(0xffffffffu, (int32_t)(ld_acquire(ptr) - target) >= 0) || wait_counter_all_slow(p, ptr, target);
}

// ---------------------------------------------------------------------------------------
// work-unit geometry

__device__ __forceinline__ int gemv_K_dev(const KParams& p, int op) {
  return op == OP_OPROJ ? p.qdim : (op == OP_DOWN ? p.F : p.d);
}

// Issue the TMA box(es) of 64-column chunk c of one GEMV stage.  Chunk layout in the
// slot: rows of the task, 128 bytes each, swizzled; QKV: first-half rows then the
// matching second-half rows of one head; gate/up: gate rows then up rows.
struct GemvBoxes {
  const void* m0;         // tensor map of the (first) matrix
  const void* m1;         // gate/up: the up matrix (its rows follow the gate rows in a chunk)
  int c1, c2;             // row coordinate; 3-D maps (QKV): head-half coordinate
  bool three_d;
  uint32_t chunk_bytes;   // one 64-column chunk of all the task's rows (128 bytes per row)
  uint32_t second_off;    // gate/up: offset of the up rows within a chunk
};

// The TMA boxes of a GEMV task's stages.  Chunk layout in the slot: the task's rows, 128
// bytes each, swizzled; QKV: first-half rows then the matching second-half rows of one head;
// gate/up: gate rows then up rows.
__device__ __forceinline__ GemvBoxes gemv_boxes(const KParams& p, const TaskDesc& t) {
  const CUtensorMapLike* maps = reinterpret_cast<const CUtensorMapLike*>(p.tmaps);
  const int n = t.nunits;
  GemvBoxes b{};
  b.chunk_bytes = (uint32_t)(n * rows_per_unit(t.op) * 128);
  b.c1 = 8 * (int)t.u0;
  switch (t.op) {
    case OP_QKV: {
      const int per_head = p.hd >> 4;
      const int hh = (int)t.u0 / per_head, m0 = (int)t.u0 - hh * per_head;
      const int mat = hh < p.nq ? 0 : (hh < p.nq + p.nkv ? 1 : 2);
      const int lh = mat == 0 ? hh : (mat == 1 ? hh - p.nq : hh - p.nq - p.nkv);
      b.m0 = maps + tmap_index(t.layer, mat, n);
      b.c1 = 8 * m0;
      b.c2 = 2 * lh;
      b.three_d = true;
      break;
    }
    case OP_GATEUP:
      b.m0 = maps + tmap_index(t.layer, 4, n);
      b.m1 = maps + tmap_index(t.layer, 5, n);
      b.second_off = (uint32_t)(8 * n * 128);
      break;
    case OP_OPROJ: b.m0 = maps + tmap_index(t.layer, 3, n); break;
    case OP_DOWN: b.m0 = maps + tmap_index(t.layer, 6, n); break;
    default: b.m0 = maps + tmap_index(p.L, 0, n); break;
  }
  return b;
}

// Split-K attention work, partitioned at run time from this step's lengths in one of two ways.
//  * Pair-aligned (whenever every (sequence i, kv head h) pair can have a range of its own):
//    the pairs of sequence i get attn_n[i] ranges each, every range one piece of attn_Ri[i]
//    tokens inside one pair.  attn_n is water-filled over the ranges: a round adds one range
//    to every pair of the sequence whose ranges are longest.  No range pays for a second
//    piece, and a pair's few pieces finish together.
//  * Otherwise the pairs are laid end to end, pair (i, h) taking ceil16(len_i) token places;
//    attention range u covers places [u R, u R + R) of that line, and its pieces are the
//    parts of the pairs it overlaps, cut at 16-token (page) boundaries, so every range holds
//    the same number of KV bytes whatever the lengths.
// A piece is the unit of split-K state (one log-sum-exp partial).
struct AttnPiece {
  int i, h;    // sequence, kv head
  int c, nc;   // piece index within the pair, pieces of the pair
  int n;       // keys of the sequence (position + 1)
  int t0, t1;  // tokens [t0, t1) of the pair, t0 a multiple of 16
};

// Piece j (in order) of range u, or false past the last one.
// QK-norm: 1/rms of head `head` (query heads first, then key heads) of batch row bi, from
// the per-unit partial sums the QKV tasks left, added in unit order.
__device__ __forceinline__ float head_inv_rms(const KParams& p, int bi, int head) {
  const int per_head = p.hd >> 4;
  const float* s = p.qkss + ((size_t)bi * (p.nq + p.nkv) + head) * per_head;
  float acc = 0.f;
  for (int u = 0; u < per_head; ++u) acc += __ldcg(s + u);
  return 1.0f / sqrtf(acc / (float)p.hd + p.eps);
}

__device__ bool attn_piece(const KParams& p, const Smem& sm, int u, int j, AttnPiece& a) {
  const int R = sm.attn_R;
  if (R == 0) {
    if (j > 0 || u >= sm.attn_u0[p.b]) return false;
    int i = 0;
    while (u >= sm.attn_u0[i + 1]) ++i;
    const int ni = sm.attn_n[i], Ri = sm.attn_Ri[i];
    const int r = u - sm.attn_u0[i];
    const int n = sm.in_len[i];
    a.i = i;
    a.h = r / ni;
    a.c = r - a.h * ni;
    a.n = n;
    a.t0 = a.c * Ri;
    if (a.t0 >= n) return false;
    a.t1 = min(a.t0 + Ri, n);
    a.nc = (n + Ri - 1) / Ri;
    return true;
  }
  const long long lo = (long long)u * R, hi = lo + R;
  long long off = 0;
  for (int i = 0; i < p.b; ++i) {
    const int n = sm.in_len[i];
    const int Lp = (n + kPage - 1) / kPage * kPage;
    const long long blk = (long long)p.nkv * Lp;
    if (off + blk > lo) {
      if (off >= hi) return false;
      const int h0 = lo > off ? (int)((lo - off) / Lp) : 0;
      const int h1 = (int)min((long long)p.nkv - 1, (hi - 1 - off) / Lp);
      for (int h = h0; h <= h1; ++h) {
        const long long st = off + (long long)h * Lp;
        const long long ts = (lo > st ? lo : st) - st, te = (hi < st + n ? hi : st + n) - st;
        if (ts >= te) continue;
        if (j-- > 0) continue;
        a.i = i;
        a.h = h;
        a.n = n;
        a.t0 = (int)ts;
        a.t1 = (int)te;
        a.c = u - (int)(st / R);
        a.nc = (int)((st + n - 1) / R - st / R) + 1;
        return true;
      }
    }
    off += blk;
  }
  return false;
}

// This step's attention partition into sm (thread 0, after the lengths were checked).  The
// pair line's range length R is the padded pair lengths spread evenly over the n_slots
// ranges, at least one full stage, and short enough that no pair is cut into more than
// kMaxChunksPerSeq pieces.
__device__ void attn_setup(const KParams& p, Smem& sm) {
  const int T = attn_stage_tokens(p.hd);
  if (p.b * p.nkv <= p.n_slots) {
    int used = p.b * p.nkv;
    for (int i = 0; i < p.b; ++i) sm.attn_n[i] = 1;
    for (;;) {
      int best = -1, bestlen = 0;
      for (int i = 0; i < p.b; ++i) {
        const int len = (sm.in_len[i] + sm.attn_n[i] - 1) / sm.attn_n[i];
        if (sm.attn_n[i] < kMaxChunksPerSeq && len > bestlen && len > T) { best = i; bestlen = len; }
      }
      if (best < 0 || used + p.nkv > p.n_slots) break;
      ++sm.attn_n[best];
      used += p.nkv;
    }
    sm.attn_u0[0] = 0;
    for (int i = 0; i < p.b; ++i) {
      const int len = (sm.in_len[i] + sm.attn_n[i] - 1) / sm.attn_n[i];
      sm.attn_Ri[i] = (len + kPage - 1) / kPage * kPage;
      sm.attn_u0[i + 1] = sm.attn_u0[i] + p.nkv * sm.attn_n[i];
    }
    sm.attn_R = 0;
    return;
  }
  long long tot = 0;
  int mx = kPage;
  for (int i = 0; i < p.b; ++i) {
    const int Lp = (sm.in_len[i] + kPage - 1) / kPage * kPage;
    tot += (long long)p.nkv * Lp;
    mx = max(mx, Lp);
  }
  long long R = (tot + p.n_slots - 1) / p.n_slots;
  R = (R + kPage - 1) / kPage * kPage;
  const long long rmin = T;
  const long long rcap = ((mx + kMaxChunksPerSeq - 3) / (kMaxChunksPerSeq - 2) + kPage - 1) / kPage * kPage;
  if (R < rmin) R = rmin;
  if (R < rcap) R = rcap;
  sm.attn_R = (int)R;
}

// ---------------------------------------------------------------------------------------
// producer warp: streams weight rows and prior KV pages into the slot ring

// Operand kind of a GEMV op: 0 x-derived (qkv, gate/up, lm head), 1 attention output (o
// projection), 2 SwiGLU output (down projection).
__device__ __forceinline__ int operand_kind(int op) { return op == OP_OPROJ ? 1 : (op == OP_DOWN ? 2 : 0); }

// The K columns [kbeg, kend) a GEMV task covers: all of K, or one K piece of a unit.
__device__ __forceinline__ void gemv_krange(const KParams& p, const TaskDesc& t, int& kbeg, int& kend) {
  kbeg = (int)t.k0 * kBoxCols;
  kend = min((int)t.k1 * kBoxCols, gemv_K_dev(p, t.op));
}

// Pool stages of a GEMV task: its columns / kc.
__device__ __forceinline__ int gemv_stages(const KParams& p, const TaskDesc& t) {
  if (t.op == OP_EMBED) return 0;
  int kbeg, kend;
  gemv_krange(p, t, kbeg, kend);
  return (kend - kbeg + t.kc - 1) / t.kc;
}

// K and V pages of stage k of attention piece a into slot `slot`: whole 16-token pages as
// tiled boxes (128-byte swizzle; head_dim 128 as [2 halves][16 rows][64]), K pages at the
// slot's start and V pages at half the slot.  Returns false on a page id out of range.
__device__ bool issue_kv(const KParams& p, Smem& sm, const TaskDesc& t, const AttnPiece& a, int k, int slot,
                         uint64_t pol) {
  const int lane = threadIdx.x & 31;
  const int T = attn_stage_tokens(p.hd);
  const int s0 = a.t0 + k * T, s1 = min(s0 + T, a.t1);
  const int pg0 = s0 / kPage, npg = (s1 - 1) / kPage - pg0 + 1;
  // a stage spans at most T / 16 <= 8 pages (ranges and stages start on page boundaries):
  // lanes 2q and 2q + 1 take the K and V box of page q, each reading its page id once
  const int q = lane >> 1;
  const bool act = q < npg;
  const int id = act ? p.ptable[a.i * p.mpps + pg0 + q] : 0;
  if (__any_sync(0xffffffffu, act && (id < 0 || id >= p.num_pages))) return false;
  const uint32_t page_bytes = (uint32_t)kPage * p.hd * 2u;
  if (lane == 0) mbar_expect_tx(&sm.wfull[slot], 2u * npg * page_bytes);
  __syncwarp();
  if (act) {
    const int row = ((t.layer * p.num_pages + id) * p.nkv + a.h) * kPage;
    uint8_t* dst = sm.pool[slot] + (size_t)(lane & 1) * T * p.hd * 2 + (size_t)q * page_bytes;
    const void* map = (lane & 1) ? (const void*)&p.vmap : (const void*)&p.kmap;
    if (p.hd == 64) tma_2d(dst, map, 0, row, &sm.wfull[slot], pol);
    else tma_3d(dst, map, 0, row, 0, &sm.wfull[slot], pol);
  }
  return true;
}

// The producer warp streams the weights and prior KV pages of the CTA's whole stream of
// stages into the slot ring, as far ahead as free slots allow: none of it depends on this
// step's activations, so it runs ahead across dependency waits and phase boundaries.
__device__ void producer(const KParams& p, Smem& sm, const TaskDesc* ts, int nt) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol = policy_evict_first();
  const int T = attn_stage_tokens(p.hd);
  uint32_t wk = 0;  // stages issued
  bool fail = false;
  for (int wt = 0; wt < nt && !fail; ++wt) {
    const TaskDesc t = ts[wt];
    if (t.op == OP_ATTN) {
      AttnPiece a;
      for (int j = 0; !fail && attn_piece(p, sm, (int)t.u0, j, a); ++j) {
        const int ns = (a.t1 - a.t0 + T - 1) / T;
        for (int k = 0; k < ns; ++k, ++wk) {
          const int slot = wk % kNumSlots;
          if (!mbar_wait_all(p, &sm.empty[slot], ((wk / kNumSlots) & 1) ^ 1)) { fail = true; break; }
          if (!issue_kv(p, sm, t, a, k, slot, pol)) {
            if (lane == 0) raise_error(p, -6 /* MK_ERR_BOUNDS */);
            fail = true;
            break;
          }
        }
      }
      continue;
    }
    // The task's boxes: map(s) and every coordinate but K are the same for all its stages,
    // so they are worked out once; a released slot then costs only its K coordinate.
    const int wn = gemv_stages(p, t);
    int kbeg, kend;
    gemv_krange(p, t, kbeg, kend);
    const GemvBoxes bx = gemv_boxes(p, t);
    for (int ws = 0; ws < wn; ++ws, ++wk) {
      const int slot = wk % kNumSlots;
      if (!mbar_wait_all(p, &sm.empty[slot], ((wk / kNumSlots) & 1) ^ 1)) { fail = true; break; }
      const int kc0 = kbeg + ws * t.kc;
      const int nch = (min((int)t.kc, kend - kc0) + kBoxCols - 1) / kBoxCols;
      if (lane == 0) mbar_expect_tx(&sm.wfull[slot], (uint32_t)nch * bx.chunk_bytes);
      __syncwarp();
      for (int c = lane; c < nch; c += 32) {
        uint8_t* dst = sm.pool[slot] + (size_t)c * bx.chunk_bytes;
        const int kk = kc0 + c * kBoxCols;
        if (bx.three_d) {
          tma_3d(dst, bx.m0, kk, bx.c1, bx.c2, &sm.wfull[slot], pol);
        } else {
          tma_2d(dst, bx.m0, kk, bx.c1, &sm.wfull[slot], pol);
          if (bx.m1) tma_2d(dst + bx.second_off, bx.m1, kk, bx.c1, &sm.wfull[slot], pol);
        }
      }
    }
  }
  if (fail) {
    // Drain: let every copy already issued land before the CTA may exit.
    if (lane == 0) {
      const uint32_t first = wk > (uint32_t)kNumSlots ? wk - kNumSlots : 0u;
      for (uint32_t s = first; s < wk; ++s) {
        const uint64_t t0 = gtimer();
        while (!mbar_try(&sm.wfull[s % kNumSlots], (s / kNumSlots) & 1))
          if (gtimer() - t0 > p.timeout_ns) break;
      }
    }
    __syncwarp();
  }
}

// The operand warp: for each GEMV task of the CTA's stream, in order, it waits for the
// dependency counter that guards the task's activations and then copies every stage's
// operand slice into the stage's slot behind the weights - per 64-column chunk one tiled box
// per bf16 (tile, part), or one box of each fp32 row for batches up to kFmaRows - completing
// on the slot's wfull barrier, whose second arrival it makes (the producer makes the first):
// the consumers then test and wait on one barrier per stage (measured 1.8 % faster at b8 than
// a barrier of its own).  Attention stages get a plain arrival.  It never waits on the
// consumers' work beyond the slot being free, so the operands of a stage are requested as
// soon as both allow.
__device__ void operand_loader(const KParams& p, Smem& sm, const TaskDesc* ts, int nt) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol = policy_evict_last();  // every SM reads the same operands
  const CUtensorMapLike* maps = reinterpret_cast<const CUtensorMapLike*>(p.tmaps);
  const int T = attn_stage_tokens(p.hd);
  const int ntile = (p.b + 7) >> 3;
  uint32_t wk = 0;  // stages handled
  bool fail = false;
  int met_ctr = -1;
  uint32_t met_target = 0;
  for (int wt = 0; wt < nt && !fail; ++wt) {
    const TaskDesc t = ts[wt];
    if (t.op == OP_EMBED) continue;
    if (t.op == OP_ATTN) {
      AttnPiece a;
      for (int j = 0; !fail && attn_piece(p, sm, (int)t.u0, j, a); ++j) {
        const int ns = (a.t1 - a.t0 + T - 1) / T;
        for (int k = 0; k < ns; ++k, ++wk) {
          const int slot = wk % kNumSlots;
          if (!mbar_wait_all(p, &sm.empty[slot], ((wk / kNumSlots) & 1) ^ 1)) { fail = true; break; }
          if (lane == 0) mbar_arrive(&sm.wfull[slot]);
          __syncwarp();
        }
      }
      continue;
    }
    // the task's activations are complete once its dependency counter is met
    if (t.wait_ctr != kNoCounter) {
      const uint32_t target = t.wait_count * p.epoch;
      if (t.wait_ctr != met_ctr || target != met_target) {
        if (!wait_counter_all(p, t.wait_ctr, t.wait_count)) { fail = true; break; }
        met_ctr = t.wait_ctr;
        met_target = target;
        if (lane == 0) asm volatile("fence.proxy.async.global;" ::: "memory");  // the copies below read it
        __syncwarp();
      }
    }
    // Everything but the K coordinate and the slot is the same for all of the task's stages:
    // worked out once.  fp32 rows (batches up to kFmaRows): per chunk c, row r's 256 bytes at
    // (c * NB + r) * 256, box e = c * NB + r.  bf16 tiles: (tile, part) q's 1024-byte box of
    // chunk c at q * kc * 16 + c * 1024, box e = q * nch + c.
    const int kind = operand_kind(t.op);
    int kbeg, kend;
    gemv_krange(p, t, kbeg, kend);
    const int R = t.nunits * rows_per_unit(t.op);
    const int nst = gemv_stages(p, t);
    const bool f32 = p.b <= kFmaRows;
    const int NB = fma_rows(p.b);
    const int rows_per_row = (kind == 0 ? p.ld_x : (kind == 1 ? p.ld_a : p.ld_h)) / 32;
    const int per_chunk = f32 ? NB : 2 * ntile;             // boxes per 64-column chunk
    const uint32_t box_bytes = f32 ? 256u : 1024u;
    const CUtensorMapLike* kmaps = maps + opmap_index(p.L, kind, 0);
    const int off0 = R * t.kc * 2;
    for (int ws = 0; ws < nst; ++ws, ++wk) {
      const int slot = wk % kNumSlots;
      if (!mbar_wait_all(p, &sm.empty[slot], ((wk / kNumSlots) & 1) ^ 1)) { fail = true; break; }
      uint8_t* dst = sm.pool[slot] + off0;
      const int k0 = kbeg + ws * t.kc;
      const int nch = (min((int)t.kc, kend - k0) + kBoxCols - 1) / kBoxCols;
      const int nbox = per_chunk * nch;
      if (lane == 0) mbar_expect_tx(&sm.wfull[slot], (uint32_t)nbox * box_bytes);
      __syncwarp();
      for (int e = lane; e < nbox; e += 32) {
        if (f32) {
          const int c = NB == 1 ? e : (e >> 1), r = e - c * NB;
          tma_2d(dst + (size_t)e * 256, kmaps + (kOpMapsPerKind - 1), 0, r * rows_per_row + k0 / 32 + 2 * c,
                 &sm.wfull[slot], pol);
        } else {
          // q = e / nch for q < 2 * kMaxTiles <= 4, without a division
          static_assert(kMaxTiles <= 2, "operand boxes of at most four (tile, part) pairs");
          const int q = (e >= nch) + (e >= 2 * nch) + (e >= 3 * nch), c = e - q * nch;
          tma_2d(dst + (size_t)q * t.kc * 16 + (size_t)c * 1024, kmaps + q, 0, k0 / 8 + 8 * c, &sm.wfull[slot], pol);
        }
      }
    }
  }
  if (fail) {
    // Drain: let every copy already issued land before the CTA may exit.
    if (lane == 0) {
      const uint32_t first = wk > (uint32_t)kNumSlots ? wk - kNumSlots : 0u;
      for (uint32_t s = first; s < wk; ++s) {
        const uint64_t t0 = gtimer();
        while (!mbar_try(&sm.wfull[s % kNumSlots], (s / kNumSlots) & 1))
          if (gtimer() - t0 > p.timeout_ns) break;
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// consumer helpers

// 1/rms of each batch row from the partial sums of squares of instance `inst`.  Each lane
// keeps eight loads in flight (partials lane + 32 (8 i + j) go to sum j), so a few hundred
// partials cost one or two L2 round trips; the order of the additions is fixed.
__device__ void compute_inv_rms(const KParams& p, Smem& sm, int inst, int nparts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* base = p.ssq + (size_t)inst * p.ssq_stride;
  for (int bi = warp; bi < p.b; bi += kConsumerWarps) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int k0 = lane; k0 < nparts; k0 += 256) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = k0 + 32 * j;
        v[j] = k < nparts ? __ldcg(base + (size_t)k * p.max_b + bi) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += v[j];
    }
    float s = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) sm.inv_rms[bi] = 1.0f / sqrtf(s / (float)p.d + p.eps);
  }
}

// Store one GEMV operand value (batch row bi, column k) in the layout this step's GEMVs read:
// fp32 rows for batches up to kFmaRows (the FMA path); else bf16 parts in the tile layout.
// Up to kTriRows batch rows, three parts (hi, mid, lo: ~24 bits, as fp32) fill the 16 rows of
// one MMA tile - hi in rows 0-3, mid in rows 4-7, lo in rows 8-11; above that, two parts (hi
// in rows 0-7, lo in rows 8-15; ~16 bits).  Each part is the bf16 rounding of what the parts
// before it left over, which is exact in fp32.
__device__ __forceinline__ void put_operand(const KParams& p, bf16* tiles, float* f, int ld, int bi, int k, float v) {
  if (p.b <= kFmaRows) {
    f[(size_t)bi * ld + opnd_row0_index(k)] = v;
    return;
  }
  const bf16 h = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h);
  const int mt = bi >> 3, row = bi & 7;
  tiles[opnd_tile_index(mt, 0, k, row, ld)] = h;
  if (p.b <= kTriRows) {
    const bf16 m = __float2bfloat16_rn(r1);
    tiles[opnd_tile_index(0, 0, k, row + 4, ld)] = m;
    tiles[opnd_tile_index(0, 1, k, row, ld)] = __float2bfloat16_rn(r1 - __bfloat162float(m));
  } else {
    tiles[opnd_tile_index(mt, 1, k, row, ld)] = __float2bfloat16_rn(r1);
  }
}

// Stream the task's stages through the eight warps and reduce into sm.ep[row][batch].
// Slot layout of a stage: the weights (per 64-column chunk: 8*G rows of 128 bytes, 16-byte
// pieces swizzled, piece c of row r at c ^ (r & 7)), then the stage's operands (opnd_*
// layouts: per bf16 (tile, part) kc * 16 bytes, or kc * 4 bytes of fp32 row 0).  Warp w takes
// the task's 32-column k blocks w, w+8, ... (counted across stages); block kb is the even (h = 0) or odd (h = 1)
// 16-byte pieces of chunk kb / 2, so lane (g, tq) reads piece 2*tq + h of row 8j + g -
// conflict-free - which holds columns 16*tq + 8*h .. +7, and the operand piece of the same
// columns at `lane` (bf16) or `tq` (fp32, shared by the 8 lanes of one tq).
// MT = 0: CUDA-core FMA on fp32 activations for NB (1 or 2 = batch) rows, the operands of
// chunk c row r at (c * NB + r) * 256 bytes; MT = 1, 2: mma.sync with MT tiles of 8 batch
// rows, the M = 16 tile holding the bf16 parts of the activations (put_operand).
// Inlined into the consumer loop like the attention body: as called functions, the two cost
// each task ~0.5-1 µs on entry (call, spills of live registers, a cold code path) and the
// step 4.7 % (b8) / 4.3 % (b1).
template <int MT, int G, int NB = 1, bool TRI = false>
__device__ __forceinline__ void gemv_body(const KParams& p, Smem& sm, const TaskDesc t, uint32_t& stage, bool& ab) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  int kbeg, kend;
  gemv_krange(p, t, kbeg, kend);
  const int kc = t.kc;
  const int nst = (kend - kbeg + kc - 1) / kc;
  constexpr int R = 8 * G;
  constexpr int NMT = MT == 0 ? 1 : MT;
  float acc[G][NMT][4];
#pragma unroll
  for (int j = 0; j < G; ++j)
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][mt][e] = 0.f;

  // every lane tests each stage's barrier one stage ahead (before the previous stage's
  // compute), a vote making the answer uniform; only a stage that had not landed by then
  // takes the blocking wait.  Waits by the whole warp - no lane-0 wait and broadcast - cut
  // 6.5 % (b8) / 7.8 % (b1) off the step over all the per-stage waits.
  bool ready = !ab && nst > 0 && __all_sync(0xffffffffu, stage_landed(sm, stage) != 0u);
  for (int s = 0; s < nst; ++s, ++stage) {
    const int slot = stage % kNumSlots;
    const uint32_t par = (stage / kNumSlots) & 1;
    if (!ab && !ready) {
      const long long w0 = (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) ? clock64() : 0ll;
      ab = !mbar_wait_all(p, &sm.wfull[slot], par);
      if (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) sm.wait_cyc += (unsigned long long)(clock64() - w0);
    }
    if (ab) continue;
    ready = s + 1 < nst && __all_sync(0xffffffffu, stage_landed(sm, stage + 1) != 0u);
    const long long tc0 = (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) ? clock64() : 0ll;
    const uint8_t* tile = sm.pool[slot];
    const uint8_t* opnd = tile + (size_t)R * kc * 2;
    const int nb = 2 * ((min(kc, kend - kbeg - s * kc) + kBoxCols - 1) / kBoxCols);
    // k block q of the task (q = s * nbs + kb) goes to warp q % 8: every warp's accumulator
    // chain covers an eighth of K whatever the stage width (tensor-core fp32 accumulation
    // truncates, so its error grows with the chain)
    const int nbs = 2 * (kc / kBoxCols);
    for (int kb = (warp + kConsumerWarps - (s * nbs) % kConsumerWarps) % kConsumerWarps; kb < nb;
         kb += kConsumerWarps) {
      const uint8_t* chunk = tile + (size_t)(kb >> 1) * (R * 128) + ((((2 * tq + (kb & 1)) ^ g)) << 4);
      uint4 A[MT == 0 ? 2 * NB : 2 * NMT];
      if constexpr (MT == 0) {
#pragma unroll
        for (int r = 0; r < NB; ++r) {
          const uint8_t* ap = opnd + ((size_t)(kb >> 1) * NB + r) * 256 + (kb & 1) * 128 + tq * 32;
          A[2 * r] = *reinterpret_cast<const uint4*>(ap);
          A[2 * r + 1] = *reinterpret_cast<const uint4*>(ap + 16);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 2 * MT; ++q)
          A[q] = *reinterpret_cast<const uint4*>(opnd + (size_t)q * kc * 16 + (size_t)kb * 512 + lane * 16);
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(chunk + (8 * j + g) * 128);
        if constexpr (MT == 0) {
#pragma unroll
          for (int r = 0; r < NB; ++r) {
            const uint4 a0 = A[2 * r], a1 = A[2 * r + 1];
            float s0 = acc[j][0][r];
            s0 = fmaf(bf_lo(w.x), __uint_as_float(a0.x), s0); s0 = fmaf(bf_hi(w.x), __uint_as_float(a0.y), s0);
            s0 = fmaf(bf_lo(w.y), __uint_as_float(a0.z), s0); s0 = fmaf(bf_hi(w.y), __uint_as_float(a0.w), s0);
            s0 = fmaf(bf_lo(w.z), __uint_as_float(a1.x), s0); s0 = fmaf(bf_hi(w.z), __uint_as_float(a1.y), s0);
            s0 = fmaf(bf_lo(w.w), __uint_as_float(a1.z), s0); s0 = fmaf(bf_hi(w.w), __uint_as_float(a1.w), s0);
            acc[j][0][r] = s0;
          }
        } else {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const uint4 H = A[2 * mt], L = A[2 * mt + 1];
            // the block's two MMAs into a fresh accumulator, added to the total in fp32
            // (round to nearest): tensor-core accumulation truncates, so no long chains
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16(d, H.x, L.x, H.y, L.y, w.x, w.y);
            mma_bf16(d, H.z, L.z, H.w, L.w, w.z, w.w);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][mt][e] += d[e];
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
    if (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) sm.tm[0] += (unsigned long long)(clock64() - tc0);
  }

  // cross-warp reduction, one 8-row batch tile at a time: red[warp][block][batch g][8 rows]
  const long long tr0 = (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) ? clock64() : 0ll;
  float* red = sm.red;
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    if (!ab) {
#pragma unroll
      for (int j = 0; j < G; ++j) {
        if constexpr (MT == 0) {
#pragma unroll
          for (int r = 0; r < NB; ++r) {
            float v = acc[j][0][r];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            if (tq == 0) red[((warp * kMaxBlocks + j) * 8 + r) * 8 + g] = v;
          }
        } else {
          float2 y = make_float2(acc[j][mt][0] + acc[j][mt][2], acc[j][mt][1] + acc[j][mt][3]);
          if constexpr (TRI) {
            // three-part activations: batch row g's mid part is D row g + 4, held by lane + 16
            y.x += __shfl_down_sync(0xffffffffu, acc[j][mt][0], 16);
            y.y += __shfl_down_sync(0xffffffffu, acc[j][mt][1], 16);
          }
          *reinterpret_cast<float2*>(&red[((warp * kMaxBlocks + j) * 8 + g) * 8 + 2 * tq]) = y;
        }
      }
    }
    cbar();
    const int nb8 = min(8, p.b - mt * 8);
    const int items = nb8 > 0 ? R * nb8 : 0;
    for (int idx = threadIdx.x; idx < items; idx += kConsumerWarps * 32) {
      const int bl = idx % nb8;
      const int row = idx / nb8;  // 8*j + r
      const int j = row >> 3, r = row & 7;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) sum += red[((w * kMaxBlocks + j) * 8 + bl) * 8 + r];
      sm.ep[row][mt * 8 + bl] = sum;
    }
    cbar();
  }
  if (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) sm.tm[1] += (unsigned long long)(clock64() - tr0);
}

// TRI (MT = 1 only): the activations are in three parts (batches up to kTriRows, put_operand).
template <int MT, int NB = 1, bool TRI = false>
__device__ void gemv_dispatch(const KParams& p, Smem& sm, const TaskDesc& t, uint32_t& stage, bool& ab, int G) {
  switch (G) {
    case 1: gemv_body<MT, 1, NB, TRI>(p, sm, t, stage, ab); break;
    case 2: gemv_body<MT, 2, NB, TRI>(p, sm, t, stage, ab); break;
    case 3: gemv_body<MT, 3, NB, TRI>(p, sm, t, stage, ab); break;
    case 4: gemv_body<MT, 4, NB, TRI>(p, sm, t, stage, ab); break;
    case 5: gemv_body<MT, 5, NB, TRI>(p, sm, t, stage, ab); break;
    case 6: gemv_body<MT, 6, NB, TRI>(p, sm, t, stage, ab); break;
    case 7: gemv_body<MT, 7, NB, TRI>(p, sm, t, stage, ab); break;
    default: gemv_body<MT, 8, NB, TRI>(p, sm, t, stage, ab); break;
  }
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

// Gain of the RMSNorm whose input the residual writer of (op, layer) produces.
__device__ __forceinline__ const bf16* next_gain(const KParams& p, int op, int layer) {
  if (op == OP_EMBED) return p.layers[0].attn_norm;
  if (op == OP_OPROJ) return p.layers[layer].mlp_norm;
  return layer + 1 < p.L ? p.layers[layer + 1].attn_norm : p.final_norm;
}

// ---------------------------------------------------------------------------------------
// consumer task bodies

// The QKV epilogue: RoPE on queries and keys (the table holds cos and sin of pos *
// inv_freq), queries to q, keys and values appended to the cache in bf16.
__device__ __forceinline__ void qkv_epilogue(const KParams& p, Smem& sm, const TaskDesc& t) {
  const int nthr = kConsumerWarps * 32;
  const int n = t.nunits;
  const int half = p.hd / 2, per_head = p.hd >> 4;
  const int hh = (int)t.u0 / per_head, m0 = (int)t.u0 - hh * per_head;
  const int items = n * 8 * p.b;
  for (int idx = threadIdx.x; idx < items; idx += nthr) {
    const int bi = idx % p.b;
    const int row = idx / p.b;  // 0 .. 8n-1 within the first half
    const int j = 8 * m0 + row;
    const float r = sm.inv_rms[bi];
    const float x1 = sm.ep[row][bi] * r;
    const float x2 = sm.ep[8 * n + row][bi] * r;
    const int pos = sm.in_pos[bi];
    if (hh < p.nq + p.nkv) {
      const float2 cs = p.rope[(size_t)pos * half + j];
      const float o1 = x1 * cs.x - x2 * cs.y;
      const float o2 = x2 * cs.x + x1 * cs.y;
      if (hh < p.nq) {
        float* qd = p.q + (size_t)bi * p.qdim + (size_t)hh * p.hd;
        qd[j] = o1;
        qd[j + half] = o2;
      } else {
        const int page = p.ptable[bi * p.mpps + pos / kPage];
        bf16* kd = p.kpool + ((((size_t)t.layer * p.num_pages + page) * p.nkv + (hh - p.nq)) * kPage +
                              pos % kPage) * p.hd;
        kd[j] = __float2bfloat16_rn(o1);
        kd[j + half] = __float2bfloat16_rn(o2);
      }
    } else {
      const int page = p.ptable[bi * p.mpps + pos / kPage];
      bf16* vd = p.vpool + ((((size_t)t.layer * p.num_pages + page) * p.nkv + (hh - p.nq - p.nkv)) * kPage +
                            pos % kPage) * p.hd;
      vd[j] = __float2bfloat16_rn(x1);
      vd[j + half] = __float2bfloat16_rn(x2);
    }
  }
}

// The QKV epilogue of a QK-norm model (Qwen3).  Per head vector, its 1/rms over head_dim is
// a common factor of all its components, so RoPE can be applied first: this task writes
// RoPE(gain * raw) for its rows - queries to q, keys to knew - and its share of the head's
// sum of squares (its units' rows of both halves, added in row order) to one slot per unit.
// Where the whole head is read (attention) the slots are added and the factor applied; the
// key is stored into the cache there.  Values are appended here as usual.
__device__ __forceinline__ void qkv_epilogue_qk_norm(const KParams& p, Smem& sm, const TaskDesc& t) {
  const int nthr = kConsumerWarps * 32;
  const int n = t.nunits;
  const int half = p.hd / 2, per_head = p.hd >> 4;
  const int hh = (int)t.u0 / per_head, m0 = (int)t.u0 - hh * per_head;
  const bool qk = hh < p.nq + p.nkv;
  if (qk)
    for (int bi = threadIdx.x; bi < p.b; bi += nthr) {
      const float r = sm.inv_rms[bi];
      float s = 0.f;
      for (int row = 0; row < 8 * n; ++row) {
        const float x1 = sm.ep[row][bi] * r, x2 = sm.ep[8 * n + row][bi] * r;
        s += x1 * x1 + x2 * x2;
      }
      float* slot = p.qkss + ((size_t)bi * (p.nq + p.nkv) + hh) * per_head + m0;
      slot[0] = s;
      for (int u = 1; u < n; ++u) slot[u] = 0.f;
    }
  const bf16* gain = !qk ? nullptr : (hh < p.nq ? p.layers[t.layer].q_norm : p.layers[t.layer].k_norm);
  const int items = n * 8 * p.b;
  for (int idx = threadIdx.x; idx < items; idx += nthr) {
    const int bi = idx % p.b;
    const int row = idx / p.b;
    const int j = 8 * m0 + row;
    const float r = sm.inv_rms[bi];
    float x1 = sm.ep[row][bi] * r;
    float x2 = sm.ep[8 * n + row][bi] * r;
    const int pos = sm.in_pos[bi];
    if (qk) {
      x1 *= __bfloat162float(gain[j]);
      x2 *= __bfloat162float(gain[j + half]);
      const float2 cs = p.rope[(size_t)pos * half + j];
      const float o1 = x1 * cs.x - x2 * cs.y;
      const float o2 = x2 * cs.x + x1 * cs.y;
      float* d = hh < p.nq ? p.q + (size_t)bi * p.qdim + (size_t)hh * p.hd
                           : p.knew + ((size_t)bi * p.nkv + (hh - p.nq)) * p.hd;
      d[j] = o1;
      d[j + half] = o2;
    } else {
      const int page = p.ptable[bi * p.mpps + pos / kPage];
      bf16* vd = p.vpool + ((((size_t)t.layer * p.num_pages + page) * p.nkv + (hh - p.nq - p.nkv)) * kPage +
                            pos % kPage) * p.hd;
      vd[j] = __float2bfloat16_rn(x1);
      vd[j + half] = __float2bfloat16_rn(x2);
    }
  }
}


__device__ void gemv_task(const KParams& p, Smem& sm, const TaskDesc& t, uint32_t& stage, bool& ab, int& inv_inst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool norm = t.op == OP_QKV || t.op == OP_GATEUP || t.op == OP_LMHEAD;
  const int inst = t.op == OP_GATEUP ? ssq_inst_oproj(t.layer)
                   : t.op == OP_QKV  ? (t.layer == 0 ? ssq_inst_embed() : ssq_inst_down(t.layer - 1))
                                     : ssq_inst_down(p.L - 1);
  // tasks of one phase share the 1/rms of their input: compute it once per phase (inv_inst is
  // the same in every consumer thread, so the barrier is taken by all or none)
  if (norm && inst != inv_inst) {
    if (!ab) compute_inv_rms(p, sm, inst, (int)t.wait_count);
    cbar();
    inv_inst = inst;
  }
  const int G = t.nunits * rows_per_unit(t.op) / 8;
  static_assert(kFmaRows == 2, "the FMA path is instantiated for 1 and 2 rows");
  if (p.b == 1) gemv_dispatch<0, 1>(p, sm, t, stage, ab, G);
  else if (p.b == 2) gemv_dispatch<0, 2>(p, sm, t, stage, ab, G);
  else if (p.b <= kTriRows) gemv_dispatch<1, 1, true>(p, sm, t, stage, ab, G);
  else if (p.b <= 8) gemv_dispatch<1>(p, sm, t, stage, ab, G);
  else gemv_dispatch<2>(p, sm, t, stage, ab, G);
  const long long te0 = (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) ? clock64() : 0ll;

  const int nthr = kConsumerWarps * 32;
  const int n = t.nunits;
  if (t.split != kNoSplit) {
    // one of the K pieces of a task group: publish this piece's sums; the last piece to
    // arrive adds all pieces' sums in piece order (the same order whoever arrives last) and
    // runs the epilogue, the others only clear their per-task partial slots
    const int rows = 8 * G;
    const int id = split_id(t.split), np = split_pieces(t.split);
    const size_t stride = (size_t)kMaxBlocks * 8 * p.max_b;  // floats per piece
    float* base = p.spart + (size_t)id * kMaxPieces * stride;
    if (!ab)
      for (int idx = threadIdx.x; idx < rows * p.b; idx += nthr) {
        const int bi = idx % p.b, row = idx / p.b;
        __stcg(base + split_piece(t.split) * stride + (size_t)row * p.max_b + bi, sm.ep[row][bi]);
      }
    cbar();
    if (threadIdx.x == 0) {
      int last = 0;
      if (!ab) {
        __threadfence();
        const uint32_t old = atom_add_acqrel(p.scnt + id, 1u);
        last = old + 1u == (uint32_t)np ? 1 : 0;
        if (last) p.scnt[id] = 0u;  // ready for the next phase
      }
      sm.flag2 = last;
    }
    cbar();
    if (!sm.flag2) {
      if (!ab && (t.op == OP_OPROJ || t.op == OP_DOWN)) {
        const int inst = t.op == OP_OPROJ ? ssq_inst_oproj(t.layer) : ssq_inst_down(t.layer);
        for (int bi = threadIdx.x; bi < p.b; bi += nthr)
          p.ssq[(size_t)inst * p.ssq_stride + (size_t)t.task_idx * p.max_b + bi] = 0.f;
      }
      if (!ab && t.op == OP_LMHEAD && p.argmax)
        for (int bi = threadIdx.x; bi < p.b; bi += nthr)
          p.lmpart[(size_t)t.task_idx * p.max_b + bi] = make_float2(-INFINITY, __int_as_float(0x7fffffff));
      if (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) sm.tm[2] += (unsigned long long)(clock64() - te0);
      return;
    }
    if (!ab)
      for (int idx = threadIdx.x; idx < rows * p.b; idx += nthr) {
        const int bi = idx % p.b, row = idx / p.b;
        const float* src = base + (size_t)row * p.max_b + bi;
        float v = __ldcg(src);
        for (int q = 1; q < np; ++q) v += __ldcg(src + q * stride);
        sm.ep[row][bi] = v;
      }
    cbar();
  }
  if (t.op == OP_QKV) {
    if (!ab && p.qk_norm) qkv_epilogue_qk_norm(p, sm, t);
    else if (!ab) qkv_epilogue(p, sm, t);
  } else if (t.op == OP_GATEUP) {
    if (!ab) {
      const int items = n * 8 * p.b;
      for (int idx = threadIdx.x; idx < items; idx += nthr) {
        const int bi = idx % p.b;
        const int row = idx / p.b;
        const float r = sm.inv_rms[bi];
        const float gv = sm.ep[row][bi] * r;
        const float uv = sm.ep[8 * n + row][bi] * r;
        put_operand(p, p.ah_t, p.ah_f, p.ld_h, bi, 8 * t.u0 + row, silu_f(gv) * uv);
      }
    }
  } else if (t.op == OP_OPROJ || t.op == OP_DOWN) {
    const int inst = t.op == OP_OPROJ ? ssq_inst_oproj(t.layer) : ssq_inst_down(t.layer);
    if (!ab) {
      const int rows = 8 * n;
      const int items = rows * p.b;
      const bf16* gain = next_gain(p, t.op, t.layer);
      float* dbg = (t.op == OP_DOWN && p.dbg) ? p.dbg + (size_t)(t.layer + 1) * p.max_b * p.d : nullptr;
      for (int idx = threadIdx.x; idx < items; idx += nthr) {
        const int bi = idx % p.b;
        const int row = idx / p.b;
        const int grow = 8 * t.u0 + row;
        float* xp = p.x + (size_t)bi * p.d + grow;
        const float xn = __ldcg(xp) + sm.ep[row][bi];
        *xp = xn;
        sm.ep[row][bi] = xn;
        put_operand(p, p.ax_t, p.ax_f, p.ld_x, bi, grow, xn * __bfloat162float(gain[grow]));
        if (dbg) dbg[(size_t)bi * p.d + grow] = xn;
      }
    }
    cbar();
    if (!ab) {
      for (int bi = warp; bi < p.b; bi += kConsumerWarps) {
        float s = 0.f;
        for (int row = lane; row < 8 * n; row += 32) s += sm.ep[row][bi] * sm.ep[row][bi];
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        // a K-split group's sum always goes to piece 0's slot: the 1/rms reduction then adds
        // the same values in the same order whichever piece finished last
        if (lane == 0) p.ssq[(size_t)inst * p.ssq_stride + (size_t)t.slot0 * p.max_b + bi] = s;
      }
    }
  } else {  // LM head
    if (!ab) {
      const int rows = 8 * n;
      const int items = rows * p.b;
      for (int idx = threadIdx.x; idx < items; idx += nthr) {
        const int bi = idx % p.b;
        const int row = idx / p.b;
        const float v = sm.ep[row][bi] * sm.inv_rms[bi];
        sm.ep[row][bi] = v;
        p.logits[(size_t)bi * p.V + 8 * t.u0 + row] = v;
      }
    }
    cbar();
    if (!ab && p.argmax) {
      for (int bi = warp; bi < p.b; bi += kConsumerWarps) {
        float best = -INFINITY;
        int bidx = 0x7fffffff;
        for (int row = lane; row < 8 * n; row += 32) {
          const float v = sm.ep[row][bi];
          if (v > best) { best = v; bidx = 8 * t.u0 + row; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, best, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
          if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
        }
        if (lane == 0) p.lmpart[(size_t)t.task_idx * p.max_b + bi] = make_float2(best, __int_as_float(bidx));
      }
      if (threadIdx.x == 0) p.lmrows[t.task_idx] = make_int2(8 * (int)t.u0, min(8 * n, p.V - 8 * (int)t.u0));
    }
  }
  if (MK_TRACE_DETAIL && p.trace && threadIdx.x == 0) sm.tm[2] += (unsigned long long)(clock64() - te0);
}

__device__ void embed_task(const KParams& p, Smem& sm, const TaskDesc& t, bool ab) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (ab) return;
  const int c0 = 8 * t.u0, nc = 8 * t.nunits;
  const bf16* gain = next_gain(p, OP_EMBED, 0);
  for (int bi = warp; bi < p.b; bi += kConsumerWarps) {
    const bf16* e = p.embed + (size_t)sm.in_tok[bi] * p.d;
    float s = 0.f;
    for (int c = lane; c < nc; c += 32) {
      const float v = __bfloat162float(e[c0 + c]);
      p.x[(size_t)bi * p.d + c0 + c] = v;
      put_operand(p, p.ax_t, p.ax_f, p.ld_x, bi, c0 + c, v * __bfloat162float(gain[c0 + c]));
      if (p.dbg) p.dbg[(size_t)bi * p.d + c0 + c] = v;
      s += v * v;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) p.ssq[(size_t)ssq_inst_embed() * p.ssq_stride + (size_t)t.task_idx * p.max_b + bi] = s;
  }
}

// Byte offset of 16-byte chunk ch (dims 8ch..8ch+7) of token row r (0..15) inside one page
// block of the pool slot: the box layout [head_dim / 64 halves][16 rows][128 bytes] with the
// 128-byte swizzle (chunk position ^= row & 7).
__device__ __forceinline__ uint32_t kv_off(int r, int ch) {
  return (uint32_t)((((ch >> 3) << 4) + r) << 7) + (uint32_t)(((ch & 7) ^ (r & 7)) << 4);
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ uint32_t split_pair(float x, float y, bool lo) {
  const float hx = __bfloat162float(__float2bfloat16_rn(x)), hy = __bfloat162float(__float2bfloat16_rn(y));
  return lo ? pack_bf16(x - hx, y - hy) : pack_bf16(hx, hy);
}

// One attention range (its pieces in turn) of GQA decode attention, flash-decode style, all
// products on tensor cores.  Per piece = (sequence i, kv head h, tokens [t0, t1)):
//   * each warp owns 16-token groups of the stages it takes (head_dim 64: all warps every
//     stage; head_dim 128: warps 0-3 even stages, 4-7 odd ones);
//   * S = Q K^T with A = the g query heads (rows 0-7 bf16 hi parts, rows 8-15 the lo
//     remainders, so q keeps ~16 mantissa bits) and B = K rows by ldmatrix;
//   * online softmax in the log2 domain, the row max shared by the 4 lanes of a row;
//   * O += P V with A = P split the same way into hi/lo rows and B = V by ldmatrix.trans;
//   * the 8 warps' (m, l, O) merge in shared memory into one log-sum-exp partial; the last
//     piece of (i, h) to finish combines all its pieces into the O-projection operand.
// QKN (QK-norm models): queries are scaled by their head's 1/rms, and the new key is
// normalised and stored here.  A template argument, so that models without QK-norm run code
// with none of it.
template <int HD, bool QKN>
__device__ __forceinline__ void attn_task(const KParams& p, Smem& sm, const TaskDesc& t, uint32_t& stage, bool& ab) {
  constexpr int T = HD == 64 ? 128 : 96;      // tokens per stage (K then V: 32 / 48 KB)
  constexpr int WPS = T / 16;                 // warps per stage, one 16-token group each
  constexpr int NG = kConsumerWarps / WPS;    // stages in flight across warp groups
  constexpr int NK = HD / 16;                 // k steps of Q K^T
  constexpr int NN = HD / 8;                  // n tiles of P V
  constexpr int PAGE = kPage * HD * 2;        // bytes of one page block
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g_ = lane >> 2, tq = lane & 3;
  const int grp = warp % WPS, wsel = warp / WPS;
  const int G = p.g;
  const float sc = 1.4426950408889634f / sqrtf((float)HD);
  const bool tr = MK_TRACE_DETAIL && p.trace && threadIdx.x == 0;
  uint32_t ks = 0;  // stage count within the task: picks the warp group
  AttnPiece a;
  for (int j = 0; attn_piece(p, sm, (int)t.u0, j, a); ++j) {
    const long long tc0 = tr ? clock64() : 0ll;
    const unsigned long long wait0 = tr ? sm.wait_cyc : 0ull;
    // Q fragments of head g_ of this kv group
    uint32_t qa[NK][4];
    {
      const bool hv = g_ < G && !ab;
      const float* qs = p.q + (size_t)a.i * p.qdim + (size_t)(a.h * G + (hv ? g_ : 0)) * HD + 2 * tq;
      const float rq = (QKN && hv) ? head_inv_rms(p, a.i, a.h * G + g_) : 1.f;
#pragma unroll
      for (int kk = 0; kk < NK; ++kk) {
        float2 v0 = make_float2(0.f, 0.f), v1 = make_float2(0.f, 0.f);
        if (hv) {
          v0 = __ldcg(reinterpret_cast<const float2*>(qs + 16 * kk));
          v1 = __ldcg(reinterpret_cast<const float2*>(qs + 16 * kk + 8));
          if (QKN) {
            v0.x *= rq; v0.y *= rq; v1.x *= rq; v1.y *= rq;
          }
        }
        qa[kk][0] = split_pair(v0.x, v0.y, false);
        qa[kk][1] = split_pair(v0.x, v0.y, true);
        qa[kk][2] = split_pair(v1.x, v1.y, false);
        qa[kk][3] = split_pair(v1.x, v1.y, true);
      }
    }
    float m_run = -INFINITY, l_run = 0.f;
    float o[NN][4];
#pragma unroll
    for (int n = 0; n < NN; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    const int newpos = a.n - 1;
    const int ns = (a.t1 - a.t0 + T - 1) / T;
    for (int k = 0; k < ns; ++k, ++stage, ++ks) {
      const int slot = stage % kNumSlots;
      if (!ab) {
        const long long w0 = tr ? clock64() : 0ll;
        ab = !mbar_wait_all(p, &sm.wfull[slot], (stage / kNumSlots) & 1);
        if (tr) sm.wait_cyc += (unsigned long long)(clock64() - w0);
      }
      const int g0 = a.t0 + k * T + 16 * grp;  // first token of this warp's group
      const int nv = min(16, a.t1 - g0);        // valid tokens in the group (<= 0: none)
      if (!ab && (int)(ks % NG) == wsel && nv > 0) {
        uint8_t* kpg = sm.pool[slot] + grp * PAGE;
        uint8_t* vpg = sm.pool[slot] + T * HD * 2 + grp * PAGE;
        bool wrote = false;
        // positions this step wrote: the row's own new token and, in a multi-token step, the
        // earlier new tokens of its sequence (rows grow0.. of the batch) - fetched before they
        // were written, so taken again from where this step's QKV tasks left them
        const int fresh = sm.in_fresh[a.i];
        const int q0 = max(fresh, g0), q1 = min(newpos, g0 + 15);
        for (int q = q0; q <= q1; ++q) {
          const int r = q - g0;
          const int page = p.ptable[a.i * p.mpps + q / kPage];
          const size_t off = ((((size_t)t.layer * p.num_pages + page) * p.nkv + a.h) * kPage + q % kPage) * HD;
          constexpr int CH = HD / 8;
          if (QKN && lane < CH) {
            // QK-norm: the key is normalised here, where the whole head vector is complete;
            // the task holding a row's own new position stores it into the cache
            const int row = sm.in_grow0[a.i] + (q - fresh);  // the batch row whose token sits at q
            const float rk = head_inv_rms(p, row, p.nq + a.h);
            const float* src = p.knew + ((size_t)row * p.nkv + a.h) * HD + lane * 8;
            const float4 f0 = __ldcg(reinterpret_cast<const float4*>(src));
            const float4 f1 = __ldcg(reinterpret_cast<const float4*>(src + 4));
            uint4 v;
            v.x = pack_bf16(f0.x * rk, f0.y * rk);
            v.y = pack_bf16(f0.z * rk, f0.w * rk);
            v.z = pack_bf16(f1.x * rk, f1.y * rk);
            v.w = pack_bf16(f1.z * rk, f1.w * rk);
            if (q == newpos) *reinterpret_cast<uint4*>(p.kpool + off + lane * 8) = v;
            *reinterpret_cast<uint4*>(kpg + kv_off(r, lane)) = v;
          } else if (lane < 2 * CH) {
            const int ch = lane % CH;
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>((lane < CH ? p.kpool : p.vpool) + off + ch * 8));
            *reinterpret_cast<uint4*>((lane < CH ? kpg : vpg) + kv_off(r, ch)) = v;
          }
          wrote = true;
        }
        if (nv < 16) {
          // rows past the sequence's end hold whatever the page held: zero their V (P is 0 there)
          for (int e = lane; e < (16 - nv) * (HD / 8); e += 32)
            *reinterpret_cast<uint4*>(vpg + kv_off(nv + e / (HD / 8), e % (HD / 8))) = make_uint4(0, 0, 0, 0);
          wrote = true;
        }
        if (wrote) {
          fence_proxy_async_smem();  // the slot is refilled by the async proxy later
          __syncwarp();
        }
        // S = Q K^T: n tile 0 = tokens 0..7, n tile 1 = tokens 8..15 of the group
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t kb = smem_u32(kpg), vb = smem_u32(vpg);
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int kk = 0; kk < NK; ++kk) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + kv_off(((mi >> 1) << 3) + rr, 2 * kk + (mi & 1)), b0, b1, b2, b3);
          mma_bf16(s0, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
          mma_bf16(s1, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
        }
        // this lane's scores of head g_: tokens 2tq, 2tq+1, 8+2tq, 9+2tq (hi row + lo row)
        float sv[4] = {(s0[0] + s0[2]) * sc, (s0[1] + s0[3]) * sc, (s1[0] + s1[2]) * sc, (s1[1] + s1[3]) * sc};
        if (2 * tq >= nv) sv[0] = -INFINITY;
        if (2 * tq + 1 >= nv) sv[1] = -INFINITY;
        if (8 + 2 * tq >= nv) sv[2] = -INFINITY;
        if (9 + 2 * tq >= nv) sv[3] = -INFINITY;
        float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m_run, mx);  // finite: token 0 of the group is valid
        const float corr = exp2f(m_run - mn);
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = exp2f(sv[e] - mn);
        l_run = l_run * corr + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
        m_run = mn;
#pragma unroll
        for (int n = 0; n < NN; ++n) {
          o[n][0] *= corr;
          o[n][1] *= corr;
          o[n][2] *= corr;
          o[n][3] *= corr;
        }
        const uint32_t pa0 = split_pair(pr[0], pr[1], false), pa1 = split_pair(pr[0], pr[1], true);
        const uint32_t pa2 = split_pair(pr[2], pr[3], false), pa3 = split_pair(pr[2], pr[3], true);
        // O += P V: B = V rows (k = the 16 tokens) transposed by ldmatrix
#pragma unroll
        for (int nn = 0; nn < NN / 2; ++nn) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + kv_off(((mi & 1) << 3) + rr, 2 * nn + (mi >> 1)), b0, b1, b2, b3);
          // this stage's P V into fresh accumulators, added to O in fp32 (round to nearest):
          // tensor-core accumulation truncates, and O lives across all the piece's stages
          float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
          mma_bf16(d0, pa0, pa1, pa2, pa3, b0, b1);
          mma_bf16(d1, pa0, pa1, pa2, pa3, b2, b3);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            o[2 * nn][e] += d0[e];
            o[2 * nn + 1][e] += d1[e];
          }
        }
      }
      __syncwarp();
      if (!ab && lane == 0) mbar_arrive(&sm.empty[slot]);
    }

    long long tr0 = 0;
    if (tr) {
      tr0 = clock64();
      sm.tm[0] += (unsigned long long)(tr0 - tc0) - (sm.wait_cyc - wait0);
    }
    // this warp's state of head g_: l summed over the row's 4 lanes, O = hi row + lo row
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if (!ab && g_ < G) {
      float* rw = sm.red + (warp * G + g_) * HD + 2 * tq;
#pragma unroll
      for (int n = 0; n < NN; ++n)
        *reinterpret_cast<float2*>(rw + 8 * n) = make_float2(o[n][0] + o[n][2], o[n][1] + o[n][3]);
      if (tq == 0) {
        sm.mw[warp][g_] = m_run;
        sm.lw[warp][g_] = l_run;
      }
    }
    cbar();
    const size_t pst = (size_t)G * (HD + 2);  // floats per piece partial
    float* pbase = p.part + ((size_t)a.i * p.nkv + a.h) * kMaxChunksPerSeq * pst;
    if (!ab) {
      float* part = pbase + (size_t)a.c * pst;
      for (int idx = threadIdx.x; idx < G * HD; idx += kConsumerWarps * 32) {
        const int h = idx / HD, dd = idx % HD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.mw[w][h]);
        float A = 0.f, Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float f = sm.mw[w][h] == -INFINITY ? 0.f : exp2f(sm.mw[w][h] - M);
          A += f * sm.red[(w * G + h) * HD + dd];
          Ls += f * sm.lw[w][h];
        }
        part[h * (HD + 2) + dd] = A;
        if (dd == 0) {
          part[h * (HD + 2) + HD] = M;
          part[h * (HD + 2) + HD + 1] = Ls;
        }
      }
    }
    cbar();
    const long long te0 = tr ? clock64() : 0ll;
    if (tr) sm.tm[1] += (unsigned long long)(te0 - tr0);
    if (threadIdx.x == 0) {
      int last = 0;
      if (!ab) {
        uint32_t* cc = p.cmb + ((size_t)t.layer * p.max_b + a.i) * p.nkv + a.h;
        const uint32_t old = atom_add_acqrel(cc, 1u);
        last = (old + 1u == (uint32_t)a.nc) ? 1 : 0;
        if (last) *cc = 0u;  // ready for the next step (every piece of (i, h) has arrived)
      }
      sm.flag2 = last;
    }
    cbar();
    if (sm.flag2) {
      // log-sum-exp combine of the nc (<= 32) piece states of (i, h): one warp per head
      // computes the weights 2^(m_c - M) / sum_c 2^(m_c - M) l_c of all pieces at once,
      // then every thread sums weighted partials with independent loads.
      float* wts = sm.red;  // [head][32]
      for (int h = warp; h < G; h += kConsumerWarps) {
        const float* pc = pbase + ((size_t)lane * G + h) * (HD + 2);
        const float mc = lane < a.nc ? __ldcg(pc + HD) : -INFINITY;
        const float lc = lane < a.nc ? __ldcg(pc + HD + 1) : 0.f;
        float M = mc;
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
        const float f = lane < a.nc ? exp2f(mc - M) : 0.f;
        float den = f * lc;
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o2);
        wts[h * 32 + lane] = f / den;
      }
      cbar();
      for (int idx = threadIdx.x; idx < G * HD; idx += kConsumerWarps * 32) {
        const int h = idx / HD, dd = idx % HD;
        const float* pc = pbase + (size_t)h * (HD + 2) + dd;
        float acc0 = 0.f, acc1 = 0.f;
        int c = 0;
        for (; c + 1 < a.nc; c += 2) {
          acc0 = fmaf(wts[h * 32 + c], __ldcg(pc + c * pst), acc0);
          acc1 = fmaf(wts[h * 32 + c + 1], __ldcg(pc + (c + 1) * pst), acc1);
        }
        if (c < a.nc) acc0 = fmaf(wts[h * 32 + c], __ldcg(pc + c * pst), acc0);
        put_operand(p, p.aa_t, p.aa_f, p.ld_a, a.i, (a.h * G + h) * HD + dd, acc0 + acc1);
      }
    }
    cbar();  // sm.red is reused by the next piece
    if (tr) sm.tm[2] += (unsigned long long)(clock64() - te0);
  }
}

// ---------------------------------------------------------------------------------------
// top-k sampling of the next token, run by the CTA that released the step's last LM-head task

// Order-preserving keys: a larger logit gives a larger key32; key64 puts the lower vocabulary
// index first among equal logits, so that all keys of one row differ and "the k largest"
// is one set.
__device__ __forceinline__ uint32_t logit_key32(float v) {
  const uint32_t u = __float_as_uint(v);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}
__device__ __forceinline__ uint64_t logit_key64(float v, int idx) {
  return ((uint64_t)logit_key32(v) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)idx);
}
__device__ __forceinline__ float key64_logit(uint64_t key) {
  const uint32_t k = (uint32_t)(key >> 32);
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}
__device__ __forceinline__ int key64_index(uint64_t key) { return (int)(0xFFFFFFFFu - (uint32_t)key); }

// The k-th largest of n keys get(0..n-1) (1 <= k <= n), found by one warp: a radix select,
// most significant 8 bits first, that stops as soon as every key left in the chosen bin is
// among the k largest (the k-th is then their minimum).  hist: 256 words of shared memory.
template <class Get>
__device__ uint64_t warp_kth_largest(Get get, int n, int k, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  uint64_t prefix = 0, mask = 0;
  uint32_t rem = (uint32_t)k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) hist[i] = 0u;
    __syncwarp();
    for (int j0 = 0; j0 < n; j0 += 32) {
      // lanes with the same digit add once (keys of one row bunch into few bins)
      const int j = j0 + lane;
      const uint64_t key = j < n ? get(j) : 0ull;
      const bool in = j < n && (key & mask) == prefix;
      const unsigned act = __ballot_sync(0xffffffffu, in);
      const unsigned digit = (unsigned)(key >> shift) & 255u;
      const unsigned peers = __match_any_sync(0xffffffffu, in ? digit : 256u + (unsigned)lane);
      if (in && lane == __ffs(peers & act) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers & act));
    }
    __syncwarp();
    // lane l holds bins 255-8l .. 248-8l: lanes in order walk the bins from the top
    uint32_t c[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) { c[q] = hist[255 - 8 * lane - q]; tot += c[q]; }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    const bool mine = excl < rem && rem <= incl;
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    uint32_t digit = 0, above = 0, inbin = 0;
    if (mine) {
      uint32_t acc = excl;
      for (int q = 0; q < 8; ++q) {
        if (acc + c[q] >= rem) { digit = 255u - 8u * lane - q; above = acc; inbin = c[q]; break; }
        acc += c[q];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    inbin = __shfl_sync(0xffffffffu, inbin, src);
    rem -= above;
    prefix |= (uint64_t)digit << shift;
    mask |= (uint64_t)255u << shift;
    __syncwarp();
    if (inbin == rem) {
      uint64_t mn = ~0ull;
      for (int j = lane; j < n; j += 32) {
        const uint64_t key = get(j);
        if ((key & mask) == prefix && key < mn) mn = key;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const uint64_t v = __shfl_xor_sync(0xffffffffu, mn, o);
        mn = v < mn ? v : mn;
      }
      return mn;
    }
  }
  return prefix;
}

// Per batch row (one warp each): the next token drawn from the top_k logits at temperature T.
//  1. Every LM-head task left its row maximum (lmpart) and its vocabulary rows (lmrows).  The
//     k largest logits all lie in the k tasks with the largest maxima: a logit of any other
//     task is below those k maxima.  So the k-th largest task maximum tau0 bounds the top k
//     from below.
//  2. The logits >= tau0 of those tasks are the candidates (shared memory; if there are more
//     than fit, the selection reads the tasks' rows from global memory instead).
//  3. The k-th largest candidate tau: the top k are the candidates >= tau, ranked by key.
//  4. Weights w_r = exp((v_r - v_0) / T) in rank order, summed in that order by one lane; the
//     token is the first rank whose running sum exceeds u * total (the last rank if rounding
//     leaves none).
__device__ __noinline__ void sample_top_k(const KParams& p, Smem& sm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // per warp: histogram, selected tasks, the top k and their weights, then keys/candidates
  constexpr int kRegion = kNumSlots * kSlotBytes / kConsumerWarps;
  uint8_t* base = &sm.pool[0][0] + (size_t)warp * kRegion;
  uint32_t* hist = reinterpret_cast<uint32_t*>(base);                       // 256 words
  int* sel = reinterpret_cast<int*>(base + 1024);                           // kMaxTopK task ids
  uint64_t* top = reinterpret_cast<uint64_t*>(base + 1024 + 4 * kMaxTopK);  // kMaxTopK keys, by rank
  float* w = reinterpret_cast<float*>(base + 1024 + 12 * kMaxTopK);          // kMaxTopK weights
  uint64_t* buf = reinterpret_cast<uint64_t*>(base + 1024 + 16 * kMaxTopK);
  const int cap = (kRegion - 1024 - 16 * kMaxTopK) / 8;
  const int n = p.n_lm_tasks;
  const int k = min(p.top_k, min(kMaxTopK, p.V));
  for (int bi = warp; bi < p.b; bi += kConsumerWarps) {
    const float2* mx = p.lmpart + bi;  // task j: mx[j * max_b]
    auto task_key = [&](int j) {
      const float2 c = __ldcg(mx + (size_t)j * p.max_b);
      return logit_key64(c.x, __float_as_int(c.y));
    };
    // 1. tau0 over the task maxima (from shared memory when they fit)
    uint64_t tau0;
    const int kt = min(k, n);
    if (n <= cap) {
      // eight loads in flight per lane
      for (int j0 = lane; j0 < n; j0 += 256) {
        float2 c[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + 32 * u;
          c[u] = j < n ? __ldcg(mx + (size_t)j * p.max_b) : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + 32 * u;
          if (j < n) buf[j] = logit_key64(c[u].x, __float_as_int(c[u].y));
        }
      }
      __syncwarp();
      tau0 = warp_kth_largest([&](int j) { return buf[j]; }, n, kt, hist);
    } else {
      tau0 = warp_kth_largest(task_key, n, kt, hist);
    }
    // the selected tasks (ties among maxima only come from tasks without a maximum of their
    // own, the pieces of a split task that did not finish it: those have no rows and are
    // skipped); at most kMaxTopK, since keys of tasks with rows all differ
    int nsel = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      bool s = false;
      if (j < n) {
        const uint64_t key = n <= cap ? buf[j] : task_key(j);
        s = key >= tau0 && isfinite(key64_logit(key));
      }
      const unsigned bal = __ballot_sync(0xffffffffu, s);
      const int at = nsel + __popc(bal & ((1u << lane) - 1u));
      if (s && at < kMaxTopK) sel[at] = j;
      nsel += __popc(bal);
    }
    nsel = min(nsel, kMaxTopK);
    __syncwarp();
    if (nsel == 0) {  // no finite logit in the row: no token (the next step rejects it as out of range)
      if (lane == 0) p.argmax[bi] = 0x7fffffff;
      continue;
    }
    // 2. candidates: the selected tasks' logits with key >= tau0.  The tasks' row ranges go to
    // shared memory first (in the space `top` takes later); then (task, row) pairs are walked
    // flat, eight loads in flight per lane
    int* row0 = reinterpret_cast<int*>(top);
    int* nrow = row0 + kMaxTopK;
    for (int s = lane; s < nsel; s += 32) {
      const int2 rr = __ldcg(p.lmrows + sel[s]);
      row0[s] = rr.x;
      nrow[s] = rr.y;
    }
    __syncwarp();
    int nc = 0;
    const int nflat = 64 * nsel;
    for (int j0 = 0; j0 < nflat; j0 += 256) {
      float v[8];
      int idx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + 32 * u + lane;
        const int s = j >> 6, r = j & 63;
        idx[u] = -1;
        v[u] = 0.f;
        if (j < nflat && r < nrow[s]) {
          idx[u] = row0[s] + r;
          v[u] = __ldcg(p.logits + (size_t)bi * p.V + idx[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint64_t key = idx[u] >= 0 ? logit_key64(v[u], idx[u]) : 0ull;
        const bool c = idx[u] >= 0 && key >= tau0;
        const unsigned bal = __ballot_sync(0xffffffffu, c);
        const int at = nc + __popc(bal & ((1u << lane) - 1u));
        if (c && at < cap) buf[at] = key;
        nc += __popc(bal);
      }
    }
    __syncwarp();
    // 3. tau = the k-th largest candidate (nc >= k: the k tasks' maxima are candidates)
    auto row_key = [&](int j) {  // the selected tasks' rows, 64 per task (padding: key 0)
      const int s = j >> 6, r = j & 63;
      const int2 rr = __ldcg(p.lmrows + sel[s]);
      if (r >= rr.y) return (uint64_t)0;
      return logit_key64(__ldcg(p.logits + (size_t)bi * p.V + rr.x + r), rr.x + r);
    };
    const bool in_smem = nc <= cap;
    const int ktop = min(k, nc);
    const uint64_t tau = in_smem ? warp_kth_largest([&](int j) { return buf[j]; }, nc, ktop, hist)
                                 : warp_kth_largest(row_key, 64 * nsel, ktop, hist);
    // the top k, unordered, then placed by rank (the number of larger keys; all keys differ)
    int nt = 0;
    const int nsrc = in_smem ? nc : 64 * nsel;
    for (int j0 = 0; j0 < nsrc; j0 += 32) {
      const int j = j0 + lane;
      const uint64_t key = j < nsrc ? (in_smem ? buf[j] : row_key(j)) : 0ull;
      const bool c = j < nsrc && key >= tau;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      const int at = nt + __popc(bal & ((1u << lane) - 1u));
      if (c && at < kMaxTopK) top[at] = key;
      nt += __popc(bal);
    }
    nt = min(nt, ktop);
    __syncwarp();
    uint64_t mine[kMaxTopK / 32];
    int rk[kMaxTopK / 32];
#pragma unroll
    for (int q = 0; q < kMaxTopK / 32; ++q) {
      const int e = 32 * q + lane;
      mine[q] = e < nt ? top[e] : 0ull;
      rk[q] = -1;
      if (e < nt) {
        int r = 0;
        for (int f = 0; f < nt; ++f) r += top[f] > mine[q] ? 1 : 0;
        rk[q] = r;
      }
    }
    __syncwarp();
#pragma unroll
    for (int q = 0; q < kMaxTopK / 32; ++q)
      if (rk[q] >= 0) top[rk[q]] = mine[q];
    __syncwarp();
    // 4. weights in rank order and the draw
    const float v0 = key64_logit(top[0]);
    for (int r = lane; r < nt; r += 32) w[r] = expf((key64_logit(top[r]) - v0) / p.temperature);
    __syncwarp();
    if (lane == 0) {
      float total = 0.f;
      for (int r = 0; r < nt; ++r) total += w[r];
      const float thr = p.uniforms[bi] * total;
      float cum = 0.f;
      int pick = nt - 1;
      for (int r = 0; r < nt; ++r) {
        cum += w[r];
        if (cum > thr) { pick = r; break; }
      }
      p.argmax[bi] = key64_index(top[pick]);
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// consumer warps: walk the stream

__device__ void consumer(const KParams& p, Smem& sm, const TaskDesc* ts, int nt) {
  uint32_t stage = 0;
  bool ab = false;
  // the last counter/target seen satisfied (counters only grow) and the ssq instance whose
  // 1/rms sm.inv_rms holds: the same in every consumer thread
  int met_ctr = -1, inv_inst = -1;
  uint32_t met_target = 0;
  for (int ti = 0; ti < nt; ++ti) {
    const TaskDesc t = ts[ti];
    // dependency wait, when the task's counter target is not met already: one thread polls,
    // the others wait at the consumer barrier
    unsigned long long tr0 = 0, tr1 = 0;
    if (threadIdx.x == 0 && p.trace) { tr0 = gtimer(); sm.wait_cyc = 0; sm.tm[0] = sm.tm[1] = sm.tm[2] = 0; }
    const uint32_t target = t.wait_count * p.epoch;
    if (t.wait_ctr != kNoCounter && (t.wait_ctr != met_ctr || target != met_target)) {
      if (threadIdx.x == 0) sm.flag = (!ab && wait_counter(p, t.wait_ctr, t.wait_count)) ? 0 : 1;
      cbar();
      ab = ab || sm.flag;
      met_ctr = t.wait_ctr;
      met_target = target;
      cbar();  // sm.flag is rewritten by the next poll
    }
    if (threadIdx.x == 0 && p.trace) tr1 = gtimer();
    switch (t.op) {
      case OP_EMBED: embed_task(p, sm, t, ab); break;
      case OP_ATTN:
        if (p.hd == 64) {
          if (p.qk_norm) attn_task<64, true>(p, sm, t, stage, ab);
          else attn_task<64, false>(p, sm, t, stage, ab);
        } else {
          if (p.qk_norm) attn_task<128, true>(p, sm, t, stage, ab);
          else attn_task<128, false>(p, sm, t, stage, ab);
        }
        break;
      default: gemv_task(p, sm, t, stage, ab, inv_inst); break;
    }
    cbar();  // every consumer write of the task is done
    if (threadIdx.x == 0) {
      // hand the task to the signal warp, which releases its counter; the consumers go on
      const int e = ti % kSigRing;
      bool ok = !ab;
      if (ti >= kSigRing) ok = mbar_wait(p, &sm.sigempty[e], ((ti / kSigRing) - 1) & 1) && ok;
      sm.sigab[e] = ok ? 0 : 1;
      mbar_arrive(&sm.sigfull[e]);
      if (p.trace) {
        unsigned long long* r = p.trace + 8ull * (p.task_off[blockIdx.x] + ti);
        r[0] = tr0;
        r[1] = tr1;
        r[2] = gtimer();
        r[3] = (unsigned long long)t.op | ((unsigned long long)t.layer << 8) |
               ((unsigned long long)blockIdx.x << 24) | (min(sm.wait_cyc, 0xFFFFFFull) << 40);
        r[4] = sm.tm[0];
        r[5] = sm.tm[1];
        r[6] = sm.tm[2];
      }
    }
  }
  // once the signal warp has released every task: if this CTA's LM-head task was the step's
  // last, reduce the per-task argmax candidates (one batch row per warp)
  if (threadIdx.x == 0 && nt > 0 && p.argmax)
    sm.flag = mbar_wait(p, &sm.sigempty[(nt - 1) % kSigRing], ((nt - 1) / kSigRing) & 1) ? sm.lm_last : 0;
  cbar();
  if (nt > 0 && p.argmax && sm.flag && p.top_k > 1) {
    sample_top_k(p, sm);
  } else if (nt > 0 && p.argmax && sm.flag) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int bi = warp; bi < p.b; bi += kConsumerWarps) {
      float best = -INFINITY;
      int bidx = 0x7fffffff;
      // eight candidates' loads in flight per lane; the comparison keeps the lowest index on ties,
      // so the order of visits does not matter
      for (int k0 = lane; k0 < p.n_lm_tasks; k0 += 256) {
        float2 c[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = k0 + 32 * u;
          c[u] = k < p.n_lm_tasks ? __ldcg(p.lmpart + (size_t)k * p.max_b + bi) : make_float2(-INFINITY, __int_as_float(0x7fffffff));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int ci = __float_as_int(c[u].y);
          if (c[u].x > best || (c[u].x == best && ci < bidx)) { best = c[u].x; bidx = ci; }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
        if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
      }
      if (lane == 0) p.argmax[bi] = bidx;
    }
  }
}

// The signal warp: for each task of the CTA's stream, in order, once the consumer warps have
// handed it over, make the task's writes visible and add one to its counter.  Generic-proxy
// writes that other SMs' bulk copies (async proxy) read next need the proxy fence; the
// release makes everything the consumers wrote before their barrier and hand-over visible to
// whoever acquires the counter.  Whether the step's last LM-head task was released here is
// left in sm.lm_last for the consumer warps.
__device__ void signaler(const KParams& p, Smem& sm, const TaskDesc* ts, int nt) {
  const int lane = threadIdx.x & 31;
  for (int ti = 0; ti < nt; ++ti) {
    const TaskDesc t = ts[ti];
    const int e = ti % kSigRing;
    if (!mbar_wait_all(p, &sm.sigfull[e], (ti / kSigRing) & 1)) break;
    int last = 0;
    if (lane == 0) {
      const long long ts0 = p.trace ? clock64() : 0ll;
      if (!sm.sigab[e]) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        if (t.op == OP_LMHEAD && p.argmax) {
          const uint32_t old = atom_add_acqrel(p.ctr + t.sig_ctr, 1u);
          last = old + 1u == (uint32_t)p.n_lm_tasks * p.epoch ? 1 : 0;
        } else {
          red_release_add(p.ctr + t.sig_ctr, 1u);  // nobody here needs the old value: no round trip
        }
      }
      if (p.trace) p.trace[8ull * (p.task_off[blockIdx.x] + ti) + 7] = (unsigned long long)(clock64() - ts0);
      if (last) sm.lm_last = 1;
      mbar_arrive(&sm.sigempty[e]);  // releases sm.lm_last to the consumers' wait
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// the kernel

__global__ void __launch_bounds__(kThreads, 1) mk_decode_kernel(const __grid_constant__ KParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kNumSlots; ++s) {
      mbar_init(&sm.wfull[s], 2);  // the producer's and the operand warp's arrivals
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    for (int e = 0; e < kSigRing; ++e) {
      mbar_init(&sm.sigfull[e], 1);
      mbar_init(&sm.sigempty[e], 1);
    }
    sm.lm_last = 0;
    fence_mbar_init();
    // scalar input checks (page ids are checked where they are used)
    int bad = 0;
    for (int i = 0; i < p.b; ++i) {
      const int tk = p.tok[i], ps = p.pos[i] + p.step_add;
      const int ln = p.lens ? p.lens[i] + p.step_add : ps + 1;
      sm.in_tok[i] = tk;
      sm.in_pos[i] = ps;
      sm.in_len[i] = ln;
      // rows of one sequence in a multi-token step: consecutive, at consecutive positions
      const int g0 = p.group_first ? p.group_first[i] : i;
      sm.in_grow0[i] = g0;
      sm.in_fresh[i] = ps;
      if (g0 < 0 || g0 > i) bad = 1;
      else if (g0 < i) {
        sm.in_fresh[i] = sm.in_fresh[g0];
        if (sm.in_grow0[g0] != g0 || ps != sm.in_pos[g0] + (i - g0)) bad = 1;
      }
      if (tk < 0 || tk >= p.V || ps < 0 || ps >= p.max_ctx || ln != ps + 1 || ps / kPage >= p.mpps) bad = 1;
      else {
        const int pg = p.ptable[i * p.mpps + ps / kPage];
        if (pg < 0 || pg >= p.num_pages) bad = 1;
      }
    }
    if (bad) raise_error(p, -6 /* MK_ERR_BOUNDS */);
    // an earlier step of a multi-step run failed: its error stands and this step does nothing
    if (ld_relaxed(&p.ctl[0]) != 0) bad = 1;
    sm.bad = bad;
    if (!bad) attn_setup(p, sm);
  }
  __syncthreads();
  if (sm.bad) return;
  const uint32_t o0 = p.task_off[blockIdx.x], o1 = p.task_off[blockIdx.x + 1];
  const int warp = threadIdx.x >> 5;
  if (warp == kProducerWarp) producer(p, sm, p.tasks + o0, (int)(o1 - o0));
  else if (warp == kOperandWarp) operand_loader(p, sm, p.tasks + o0, (int)(o1 - o0));
  else if (warp == kSignalWarp) signaler(p, sm, p.tasks + o0, (int)(o1 - o0));
  else consumer(p, sm, p.tasks + o0, (int)(o1 - o0));
}

// RoPE table: (cos, sin) of pos * inv_freq_j, computed in double, stored as fp32.
__global__ void rope_table_kernel(float2* table, int max_ctx, int hd, const RopeFreq f) {
  const int half = hd / 2;
  const long long n = (long long)max_ctx * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int pos = (int)(idx / half), j = (int)(idx % half);
    const double inv = f.inv_freq[j];
    double sn, cs;
    sincos((double)pos * inv, &sn, &cs);
    table[idx] = make_float2((float)cs, (float)sn);
  }
}

cudaError_t launch_decode(const KParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = sizeof(Smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // co-residency of all CTAs (no grid sync is used)
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mk_decode_kernel, p);
}

cudaError_t launch_rope_table(float2* table, int max_ctx, int hd, const RopeFreq& f, cudaStream_t s) {
  rope_table_kernel<<<256, 256, 0, s>>>(table, max_ctx, hd, f);
  return cudaGetLastError();
}

cudaError_t kernel_attributes(int* regs, int* local_bytes, int* max_threads) {
  cudaError_t e = cudaFuncSetAttribute(mk_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(Smem));
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, mk_decode_kernel);
  if (e != cudaSuccess) return e;
  if (regs) *regs = fa.numRegs;
  if (local_bytes) *local_bytes = (int)fa.localSizeBytes;
  if (max_threads) *max_threads = fa.maxThreadsPerBlock;
  return cudaSuccess;
}

}  // namespace mk
