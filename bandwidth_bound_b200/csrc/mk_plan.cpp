// Per-SM instruction streams for the decode megakernel, and their static validator.
//
// The pages' structure ("ForgeMegakernel", §4.1: per-SM instruction streams,
// dependency counters instead of grid-wide barriers; the AutoMegaKernel summary:
// a static validator proves the schedule deadlock-free and race-free before it
// runs; "Inside the megakernel serving engine": idle SMs take ready work instead
// of waiting on a wave) is realised here as plain host code:
//  * every GEMV phase (per layer qkv / oproj / gateup / down, lm head) ends at a
//    counter that every SM waits on, so its slowest SM sets the pace.  The phase takes
//    the cheaper, by a cost model of bytes plus a fixed cost per task and per K piece,
//    of equal ranges of (unit, 64-column chunk) work - a unit group that a range
//    boundary cuts becomes K pieces whose partial sums the last to finish adds - and
//    one task per SM (row groups within one unit of each other, each cut into equal K
//    pieces); the attention phase is cut into equal token ranges at run time;
//  * each task waits on exactly one counter (all tasks of the phase it reads)
//    and adds one to its own phase's counter.
#include "mk_plan.h"

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <numeric>

namespace mk {

// GEMV phases with less than this many weight bytes per SM keep whole units per task in the
// equal-range partition.
constexpr long long kSplitMinBytes = 512 * 1024;

// The plan's cost model for choosing among partitions of a GEMV phase: every phase ends at
// a counter all SMs wait on, so the estimate that matters is the slowest SM's - its weight
// and operand bytes plus a fixed cost per task (reduction, epilogue, release, and the pool
// standing full meanwhile; measured ~7-9 us per extra task at batch 8) and per K piece
// (partial sums written, counted and re-read), both in byte equivalents.
constexpr long long kTaskCostBytes = 256 * 1024;
constexpr long long kPieceCostBytes = 96 * 1024;

// One candidate partition of a GEMV phase: (SM, task) pairs in creation order (a split
// group's piece 0 before its other pieces), task_idx and slot0 still unset; split ids 0..nids-1.
struct Cand {
  std::vector<std::pair<int, TaskDesc>> tasks;
  int nids = 0;
};

Geometry geometry(const mk_model_cfg& c) {
  Geometry G;
  G.L = c.n_layers;
  G.d = c.hidden;
  G.nq = c.n_heads;
  G.nkv = c.n_kv_heads;
  G.hd = c.head_dim;
  G.F = c.ffn;
  G.V = c.vocab;
  G.g = c.n_kv_heads > 0 ? c.n_heads / c.n_kv_heads : 0;
  G.qdim = c.n_heads * c.head_dim;
  G.kvdim = c.n_kv_heads * c.head_dim;
  return G;
}

int gemv_K(const Geometry& G, int op) {
  switch (op) {
    case OP_QKV: case OP_GATEUP: case OP_LMHEAD: return G.d;
    case OP_OPROJ: return G.qdim;
    case OP_DOWN: return G.F;
    default: return 0;
  }
}

int phase_units(const Geometry& G, int op) {
  switch (op) {
    case OP_EMBED: return G.d / 8;
    case OP_QKV: return (G.nq + 2 * G.nkv) * (G.hd / 16);
    case OP_OPROJ: case OP_DOWN: return G.d / 8;
    case OP_GATEUP: return G.F / 8;
    case OP_LMHEAD: return G.V / 8;
    default: return 0;
  }
}

long long unit_weight_bytes(const Geometry& G, int op) {
  if (op == OP_EMBED || op == OP_ATTN) return 0;
  return (long long)rows_per_unit(op) * gemv_K(G, op) * 2;
}

static bool set_err(std::string* err, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static bool set_err(std::string* err, const char* fmt, ...) {
  if (err) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    *err = buf;
  }
  return false;
}

int check_cfg(const mk_model_cfg& c, std::string* err) {
  if (c.n_layers < 1 || c.hidden < 8 || c.n_heads < 1 || c.n_kv_heads < 1 || c.ffn < 8 || c.vocab < 8 ||
      c.max_batch < 1 || c.max_ctx < 1) {
    set_err(err, "model cfg: sizes must be positive");
    return MK_ERR_INVALID_ARG;
  }
  if (!(c.rms_eps > 0.f) || !(c.rope_theta > 1.f)) {
    set_err(err, "model cfg: rms_eps must be > 0 and rope_theta > 1");
    return MK_ERR_INVALID_ARG;
  }
  if (c.rope_scale_factor > 1.f &&
      !(c.rope_low_freq_factor > 0.f && c.rope_high_freq_factor > c.rope_low_freq_factor &&
        c.rope_original_max_pos > 0)) {
    set_err(err, "model cfg: RoPE scaling needs 0 < low_freq_factor < high_freq_factor and original_max_pos > 0");
    return MK_ERR_INVALID_ARG;
  }
  if (c.qk_norm != 0 && c.qk_norm != 1) { set_err(err, "model cfg: qk_norm must be 0 or 1"); return MK_ERR_INVALID_ARG; }
  if (c.page_size != kPage) { set_err(err, "page_size must be %d", kPage); return MK_ERR_UNSUPPORTED_CFG; }
  if (c.head_dim != 64 && c.head_dim != 128) { set_err(err, "head_dim must be 64 or 128"); return MK_ERR_UNSUPPORTED_CFG; }
  if (c.n_heads % c.n_kv_heads) { set_err(err, "n_heads must be a multiple of n_kv_heads"); return MK_ERR_UNSUPPORTED_CFG; }
  int g = c.n_heads / c.n_kv_heads;
  if (g > 8 || (c.head_dim == 128 && g > 4)) {
    set_err(err, "query heads per kv head: at most 8 (4 at head_dim 128)");
    return MK_ERR_UNSUPPORTED_CFG;
  }
  if (c.hidden % 8 || c.ffn % 8 || c.vocab % 8) {
    set_err(err, "hidden, ffn and vocab must be multiples of 8");
    return MK_ERR_UNSUPPORTED_CFG;
  }
  if (c.max_batch > kMaxBatch) { set_err(err, "max_batch must be <= %d", kMaxBatch); return MK_ERR_UNSUPPORTED_CFG; }
  if (c.max_ctx > 65536) { set_err(err, "max_ctx must be <= 65536"); return MK_ERR_UNSUPPORTED_CFG; }
  if (c.hidden > 65535 * 8 || c.ffn > 65535 || c.hidden > 65535) {
    set_err(err, "hidden and ffn must fit the descriptor's 16-bit stage width");
    return MK_ERR_UNSUPPORTED_CFG;
  }
  return MK_OK;
}

// Phase order of one step: embed, per layer qkv attn oproj gateup down, lm head.
struct PhaseRef {
  int op, layer;
};

static std::vector<PhaseRef> phase_order(int L) {
  std::vector<PhaseRef> v;
  v.push_back({OP_EMBED, 0});
  for (int l = 0; l < L; ++l)
    for (int op : {OP_QKV, OP_ATTN, OP_OPROJ, OP_GATEUP, OP_DOWN}) v.push_back({op, l});
  v.push_back({OP_LMHEAD, 0});
  return v;
}

static int sig_counter(int op, int layer, int L) {
  switch (op) {
    case OP_EMBED: return ctr_embed();
    case OP_QKV: return ctr_layer(layer, 0);
    case OP_ATTN: return ctr_layer(layer, 1);
    case OP_OPROJ: return ctr_layer(layer, 2);
    case OP_GATEUP: return ctr_layer(layer, 3);
    case OP_DOWN: return ctr_layer(layer, 4);
    case OP_LMHEAD: return ctr_lm(L);
  }
  return -1;
}

// The counter a phase waits on: the phase whose output it reads first.
static int wait_counter(int op, int layer, int L) {
  switch (op) {
    case OP_EMBED: return kNoCounter;
    case OP_QKV: return layer == 0 ? ctr_embed() : ctr_layer(layer - 1, 4);
    case OP_ATTN: return ctr_layer(layer, 0);
    case OP_OPROJ: return ctr_layer(layer, 1);
    case OP_GATEUP: return ctr_layer(layer, 2);
    case OP_DOWN: return ctr_layer(layer, 3);
    case OP_LMHEAD: return ctr_layer(L - 1, 4);
  }
  return kNoCounter;
}

int build_plan(const mk_model_cfg& c, const mk_plan_opts* opts, mk_plan_s* P, std::string* err) {
  int rc = check_cfg(c, err);
  if (rc) return rc;
  const Geometry G = geometry(c);
  P->cfg = c;
  P->num_sms = (opts && opts->num_sms > 0) ? opts->num_sms : 148;
  P->attn_slots_per_sm = (opts && opts->attn_slots_per_sm > 0) ? opts->attn_slots_per_sm : 1;
  P->max_blocks = (opts && opts->max_blocks > 0) ? opts->max_blocks : kMaxBlocks;
  if (P->num_sms > 4096 || P->attn_slots_per_sm > 64 || P->max_blocks > kMaxBlocks) {
    set_err(err, "plan options out of range");
    return MK_ERR_INVALID_ARG;
  }
  const int S = P->num_sms * P->attn_slots_per_sm;
  if (S > 65535) { set_err(err, "too many attention slots"); return MK_ERR_INVALID_ARG; }
  const int nsm = P->num_sms;
  P->streams.assign(nsm, {});
  P->signalers.assign(num_counters(G.L), 0);
  P->max_phase_tasks = 0;
  std::vector<long long> cum(nsm, 0);

  std::vector<PhaseRef> order = phase_order(G.L);
  std::vector<int> phase_tasks(order.size(), 0);
  // First pass: place units; wait counts need the task count of the awaited phase,
  // which always comes earlier in the order, so one pass suffices.
  std::vector<int> tasks_of_counter(num_counters(G.L), 0);
  for (size_t pi = 0; pi < order.size(); ++pi) {
    const int op = order[pi].op, l = order[pi].layer;
    const int sig = sig_counter(op, l, G.L);
    const int wc = wait_counter(op, l, G.L);
    const uint32_t wcount = wc == kNoCounter ? 0u : (uint32_t)tasks_of_counter[wc];
    int tidx = 0;
    if (op == OP_ATTN) {
      for (int sm = 0; sm < nsm; ++sm)
        for (int s = 0; s < P->attn_slots_per_sm; ++s) {
          TaskDesc t{};
          t.op = OP_ATTN;
          t.nunits = 1;
          t.layer = (uint16_t)l;
          t.u0 = (uint32_t)(s * nsm + sm);
          t.task_idx = (uint16_t)tidx++;
          t.kc = 0;
          t.wait_ctr = (uint16_t)wc;
          t.wait_count = wcount;
          t.sig_ctr = (uint16_t)sig;
          P->streams[sm].push_back(t);
        }
    } else if (op == OP_EMBED) {
      const int U = phase_units(G, op);
      for (int sm = 0, u = 0; sm < nsm; ++sm) {
        const int n = U / nsm + (sm < U % nsm ? 1 : 0);
        if (n == 0) continue;
        TaskDesc t{};
        t.op = (uint8_t)op;
        t.nunits = (uint8_t)n;
        t.u0 = (uint32_t)u;
        t.task_idx = (uint16_t)tidx++;
        t.wait_ctr = (uint16_t)wc;
        t.sig_ctr = (uint16_t)sig;
        t.split = kNoSplit;
        t.slot0 = t.task_idx;
        P->streams[sm].push_back(t);
        u += n;
      }
    } else {
      const int U = phase_units(G, op);
      const int K = gemv_K(G, op);
      const int nkb = (K + kBoxCols - 1) / kBoxCols;
      const int rpu = rows_per_unit(op);
      const int seg = op == OP_QKV ? G.hd / 16 : U;  // QKV tasks stay inside one head
      const int mu = std::max(1, std::min(max_units(op), P->max_blocks * 8 / rpu));
      auto make_task = [&](int u0, int n, int k0, int k1) {
        TaskDesc t{};
        t.op = (uint8_t)op;
        t.nunits = (uint8_t)n;
        t.layer = (uint16_t)l;
        t.u0 = (uint32_t)u0;
        t.k0 = (uint16_t)k0;
        t.k1 = (uint16_t)k1;
        t.split = kNoSplit;
        const int cols = std::min(k1 * kBoxCols, K) - k0 * kBoxCols;
        t.kc = (uint16_t)stage_cols(n * rpu / 8, cols, c.max_batch);
        t.wait_ctr = (uint16_t)wc;
        t.wait_count = wcount;
        t.sig_ctr = (uint16_t)sig;
        return t;
      };
      auto task_cost = [&](const TaskDesc& t) {
        const long long cols = std::min((int)t.k1 * kBoxCols, K) - (long long)t.k0 * kBoxCols;
        return (long long)t.nunits * rpu * cols * 2 + cols * operand_col_bytes(c.max_batch) + kTaskCostBytes +
               (t.split != kNoSplit ? kPieceCostBytes : 0);
      };
      auto cand_cost = [&](const Cand& cd) {
        std::vector<long long> per(nsm, 0);
        for (const auto& st : cd.tasks) per[st.first] += task_cost(st.second);
        return *std::max_element(per.begin(), per.end());
      };
      std::vector<Cand> cands;

      // (1) Equal ranges.  Units are grouped into tasks of <= max_u units (QKV groups inside
      // one head); the work is the line of (group, 64-column chunk) pairs weighted by the
      // group's units, cut into equal ranges, one per SM.  A group that a cut falls into
      // becomes K pieces (<= kMaxPieces), each with all of the group's rows; the last piece
      // to finish adds the partial sums.
      {
        Cand cd;
        // groups small enough that every SM gets work and no group needs more than kMaxPieces
        const int max_u = std::max(1, std::min({max_units(op), P->max_blocks * 8 / rpu, (kMaxPieces - 1) * U / nsm}));
        std::vector<std::pair<int, int>> groups;  // (u0, n)
        for (int x = 0; x < U;) {
          const int y = std::min(U, (x / seg + 1) * seg);
          const int len = y - x, ng = (len + max_u - 1) / max_u;
          for (int k = 0, v = x; k < ng; ++k) {
            const int nk = len / ng + (k < len % ng ? 1 : 0);
            groups.push_back({v, nk});
            v += nk;
          }
          x = y;
        }
        const long long W = (long long)U * nkb;
        if ((long long)U * unit_weight_bytes(G, op) / nsm < kSplitMinBytes) {
          // a small phase: whole units only, each SM a contiguous range of U / nsm or
          // U / nsm + 1 units cut into tasks of <= max_units units inside head segments; the
          // extra units of the phase go to the SMs with the fewest bytes so far
          std::vector<int> cnt(nsm, U / nsm), idx(nsm);
          std::iota(idx.begin(), idx.end(), 0);
          std::stable_sort(idx.begin(), idx.end(), [&](int a2, int b2) { return cum[a2] < cum[b2]; });
          for (int k = 0; k < U % nsm; ++k) cnt[idx[k]]++;
          for (int sm = 0, u = 0; sm < nsm; ++sm) {
            const int n = cnt[sm];
            for (int a2 = u, end = u + n; a2 < end;) {
              const int b2 = std::min(end, (a2 / seg + 1) * seg);
              const int len = b2 - a2, ntask = (len + mu - 1) / mu;
              for (int k = 0, v = a2; k < ntask; ++k) {
                const int nk = len / ntask + (k < len % ntask ? 1 : 0);
                cd.tasks.push_back({sm, make_task(v, nk, 0, nkb)});
                v += nk;
              }
              a2 = b2;
            }
            u += n;
          }
        } else {
          const long long gmax = (long long)max_u * nkb;
          // ranges long enough that no group falls into more than kMaxPieces of them
          const int nuse = (int)std::max<long long>(1, std::min<long long>(nsm, W * (kMaxPieces - 1) / gmax));
          std::vector<long long> cut(nuse + 1);
          {
            // cuts at chunk boundaries of the group they fall into
            long long pos = 0;
            size_t gi = 0;
            cut[0] = 0;
            for (int s2 = 1; s2 < nuse; ++s2) {
              const long long want = W * s2 / nuse;
              while (gi < groups.size() && pos + (long long)groups[gi].second * nkb <= want) {
                pos += (long long)groups[gi].second * nkb;
                ++gi;
              }
              const long long within = want - pos;  // inside group gi
              const int n = gi < groups.size() ? groups[gi].second : 1;
              cut[s2] = pos + (within / n) * n;
            }
            cut[nuse] = W;
          }
          // per group: its start on the line, and the ranges (pieces) it falls into
          std::vector<long long> gstart(groups.size() + 1, 0);
          for (size_t g = 0; g < groups.size(); ++g) gstart[g + 1] = gstart[g] + (long long)groups[g].second * nkb;
          std::vector<int> gid(groups.size(), -1), gpieces(groups.size(), 1);
          for (size_t g = 0; g < groups.size(); ++g) {
            int np = 0;
            for (int s2 = 0; s2 < nuse; ++s2)
              if (cut[s2] < gstart[g + 1] && cut[s2 + 1] > gstart[g]) ++np;
            gpieces[g] = np;
            if (np > 1) gid[g] = cd.nids++;
          }
          for (int s2 = 0; s2 < nuse; ++s2) {
            const long long a2 = cut[s2], b2 = cut[s2 + 1];
            if (a2 >= b2) continue;
            for (size_t g = 0; g < groups.size(); ++g) {
              if (gstart[g + 1] <= a2 || gstart[g] >= b2) continue;
              const int n = groups[g].second;
              const int k0 = (int)((std::max(a2, gstart[g]) - gstart[g]) / n);
              const int k1 = (int)((std::min(b2, gstart[g + 1]) - gstart[g]) / n);
              if (k0 >= k1) continue;
              TaskDesc t = make_task(groups[g].first, n, k0, k1);
              if (gpieces[g] > 1) {
                int piece = 0;
                for (int s3 = 0; s3 < s2; ++s3)
                  if (cut[s3] < gstart[g + 1] && cut[s3 + 1] > gstart[g] && cut[s3] < cut[s3 + 1]) ++piece;
                t.split = split_tag(gid[g], piece, gpieces[g]);
              }
              cd.tasks.push_back({s2, t});
            }
          }
        }
        cands.push_back(std::move(cd));
      }

      // (2) One task per SM: n row groups whose sizes differ by at most one unit (QKV: a
      // head's units split among its groups), each cut into m equal K pieces, n * m <= nsm.
      // Slightly unequal bytes, but no SM pays for a second task.
      for (int m = 1; m <= kMaxPieces && m <= nkb; ++m) {
        const int n = nsm / m;
        const int nseg = (U + seg - 1) / seg;
        if (n < nseg) continue;
        std::vector<std::pair<int, int>> groups;  // (u0, n)
        bool ok = true;
        for (int sg = 0; sg < nseg && ok; ++sg) {
          const int x = sg * seg, len = std::min(U, x + seg) - x;
          // this segment's share of the n groups, by its units
          const int g_lo = (int)((long long)n * x / U), g_hi = (int)((long long)n * (x + len) / U);
          const int ng = std::min(len, std::max(1, g_hi - g_lo));
          if ((len + ng - 1) / ng > mu) { ok = false; break; }
          for (int k = 0, v = x; k < ng; ++k) {
            const int nk = len / ng + (k < len % ng ? 1 : 0);
            groups.push_back({v, nk});
            v += nk;
          }
        }
        if (!ok || (int)groups.size() * m > nsm) continue;
        Cand cd;
        for (const auto& gr : groups) {
          const int id = m > 1 ? cd.nids++ : -1;
          for (int q = 0; q < m; ++q) {
            const int k0 = nkb * q / m, k1 = nkb * (q + 1) / m;
            TaskDesc t = make_task(gr.first, gr.second, k0, k1);
            if (m > 1) t.split = split_tag(id, q, m);
            cd.tasks.push_back({0, t});
          }
        }
        // the largest tasks to the SMs with the fewest bytes so far, keeping the step's
        // totals level (task order, and so piece order, is unchanged)
        std::vector<int> ti(cd.tasks.size()), si(nsm);
        std::iota(ti.begin(), ti.end(), 0);
        std::iota(si.begin(), si.end(), 0);
        std::stable_sort(ti.begin(), ti.end(), [&](int x, int y) {
          return task_cost(cd.tasks[x].second) > task_cost(cd.tasks[y].second);
        });
        std::stable_sort(si.begin(), si.end(), [&](int x, int y) { return cum[x] < cum[y]; });
        for (size_t k = 0; k < ti.size(); ++k) cd.tasks[ti[k]].first = si[k];
        cands.push_back(std::move(cd));
      }

      size_t best = 0;
      for (size_t k = 1; k < cands.size(); ++k)
        if (cand_cost(cands[k]) < cand_cost(cands[best])) best = k;
      const Cand& cd = cands[best];
      std::vector<int> slot0_of(cd.nids, -1);
      for (const auto& st : cd.tasks) {
        TaskDesc t = st.second;
        t.task_idx = (uint16_t)tidx++;
        t.slot0 = t.task_idx;
        if (t.split != kNoSplit) {
          const int id = split_id(t.split);
          if (split_piece(t.split) == 0) slot0_of[id] = t.task_idx;  // piece 0 comes first
          t.slot0 = (uint16_t)slot0_of[id];
        }
        P->streams[st.first].push_back(t);
        const int cols = std::min((int)t.k1 * kBoxCols, K) - (int)t.k0 * kBoxCols;
        cum[st.first] += (long long)t.nunits * rpu * cols * 2;
      }
      P->max_split_ids = std::max(P->max_split_ids, cd.nids);
    }
    phase_tasks[pi] = tidx;
    tasks_of_counter[sig] += tidx;
    P->signalers[sig] += tidx;
    if (op != OP_ATTN) P->max_phase_tasks = std::max(P->max_phase_tasks, tidx);
    if (op == OP_LMHEAD) P->n_lm_tasks = tidx;
  }
  return MK_OK;
}

// ---------------------------------------------------------------------------------------
// Validator

namespace {

// X: fp32 residual; AX: its normalised-gain operand for the next GEMV; AA: attention
// output operand; AH: SwiGLU output operand.
enum Buf { B_X, B_Q, B_ATTN, B_H, B_PART, B_LOGITS, B_LMPART, B_KVNEW, B_SSQ, B_AX, B_SPLIT };

struct Access {
  int buf, inst;   // inst: layer for KVNEW, ssq instance for SSQ, 0 otherwise
  bool write;
};

std::vector<Access> accesses_of_phase(int op, int l, int L) {
  switch (op) {
    case OP_EMBED: return {{B_X, 0, true}, {B_AX, 0, true}, {B_SSQ, ssq_inst_embed(), true}};
    case OP_QKV:
      return {{B_AX, 0, false}, {B_SSQ, l == 0 ? ssq_inst_embed() : ssq_inst_down(l - 1), false},
              {B_Q, 0, true}, {B_KVNEW, l, true}};
    case OP_ATTN: return {{B_Q, 0, false}, {B_KVNEW, l, false}, {B_PART, 0, true}, {B_ATTN, 0, true}};
    case OP_OPROJ:
      return {{B_ATTN, 0, false}, {B_X, 0, true}, {B_AX, 0, true}, {B_SSQ, ssq_inst_oproj(l), true}};
    case OP_GATEUP: return {{B_AX, 0, false}, {B_SSQ, ssq_inst_oproj(l), false}, {B_H, 0, true}};
    case OP_DOWN:
      return {{B_H, 0, false}, {B_X, 0, true}, {B_AX, 0, true}, {B_SSQ, ssq_inst_down(l), true}};
    case OP_LMHEAD:
      return {{B_AX, 0, false}, {B_SSQ, ssq_inst_down(L - 1), false}, {B_LOGITS, 0, true}, {B_LMPART, 0, true}};
  }
  return {};
}

std::vector<Access> accesses(int op, int l, int L) {
  std::vector<Access> v = accesses_of_phase(op, l, L);
  if (op != OP_EMBED && op != OP_ATTN) v.push_back({B_SPLIT, 0, true});  // K-piece partials and counters
  return v;
}

}  // namespace

int validate_plan(const mk_plan_s& p, std::string* err) {
  std::string e;
  if (check_cfg(p.cfg, &e) != MK_OK) { set_err(err, "%s", e.c_str()); return MK_ERR_SCHEDULE_INVALID; }
  const Geometry G = geometry(p.cfg);
  const int nsm = (int)p.streams.size();
  const int nctr = num_counters(G.L);
  const int S = p.num_sms * p.attn_slots_per_sm;
  std::vector<PhaseRef> order = phase_order(G.L);
  auto phase_index = [&](int op, int l) -> int {
    if (op == OP_EMBED) return 0;
    if (op == OP_LMHEAD) return (int)order.size() - 1;
    int k = op == OP_QKV ? 0 : op == OP_ATTN ? 1 : op == OP_OPROJ ? 2 : op == OP_GATEUP ? 3 : 4;
    return 1 + 5 * l + k;
  };
  const int NP = (int)order.size();

  // 1. each task well formed; units covered exactly once (a unit cut into K pieces: its two
  // pieces tile its chunks, carry the same boundary and pieces 0 and 1); stages fit a slot
  std::vector<std::vector<int>> cover(NP);
  struct Piece { int k0, k1, split, u0, n; };
  std::vector<std::vector<std::vector<Piece>>> pieces(NP);
  for (int pi = 0; pi < NP; ++pi) {
    int op = order[pi].op;
    cover[pi].assign(op == OP_ATTN ? S : phase_units(G, op), 0);
    pieces[pi].assign(cover[pi].size(), {});
  }
  std::vector<int> n_sig(nctr, 0);
  std::vector<int> phase_of_sig(nctr, -1);
  for (int sm = 0; sm < nsm; ++sm)
    for (size_t k = 0; k < p.streams[sm].size(); ++k) {
      const TaskDesc& t = p.streams[sm][k];
      if (t.op < OP_EMBED || t.op > OP_LMHEAD || t.layer >= G.L) {
        set_err(err, "sm %d task %zu: bad op %d / layer %d", sm, k, t.op, t.layer);
        return MK_ERR_SCHEDULE_INVALID;
      }
      int pi = phase_index(t.op, t.layer);
      if (t.nunits < 1 || t.u0 + t.nunits > cover[pi].size()) {
        set_err(err, "sm %d task %zu (op %d layer %d): units [%u, %u) outside [0, %zu)", sm, k, t.op,
                t.layer, t.u0, t.u0 + t.nunits, cover[pi].size());
        return MK_ERR_SCHEDULE_INVALID;
      }
      const bool gemv = t.op != OP_EMBED && t.op != OP_ATTN;
      const int nkb = gemv ? (gemv_K(G, t.op) + kBoxCols - 1) / kBoxCols : 0;
      if (gemv && (t.k0 >= t.k1 || t.k1 > nkb)) {
        set_err(err, "sm %d task %zu: K chunks [%d, %d) outside [0, %d)", sm, k, t.k0, t.k1, nkb);
        return MK_ERR_SCHEDULE_INVALID;
      }
      if (gemv && (t.split != kNoSplit || t.k0 != 0 || t.k1 != nkb)) {
        if (t.split == kNoSplit || split_id(t.split) >= p.max_split_ids) {
          set_err(err, "sm %d task %zu: a K piece without a valid split tag", sm, k);
          return MK_ERR_SCHEDULE_INVALID;
        }
        for (uint32_t u = t.u0; u < t.u0 + t.nunits; ++u)
          pieces[pi][u].push_back({t.k0, t.k1, t.split, (int)t.u0, t.nunits});
      } else {
        for (uint32_t u = t.u0; u < t.u0 + t.nunits; ++u) cover[pi][u]++;
      }
      if (gemv) {
        const int rows = t.nunits * rows_per_unit(t.op);
        const int K = std::min((int)t.k1 * kBoxCols, gemv_K(G, t.op)) - (int)t.k0 * kBoxCols;
        if (t.nunits > max_units(t.op)) {
          set_err(err, "sm %d task %zu: %d rows exceed %d", sm, k, rows, kMaxBlocks * 8);
          return MK_ERR_SCHEDULE_INVALID;
        }
        if (t.kc < kBoxCols || t.kc % kBoxCols || t.kc > round_up(K, kBoxCols) ||
            (long long)t.kc * (rows * 2 + operand_col_bytes(p.cfg.max_batch)) > kSlotBytes) {
          set_err(err, "sm %d task %zu: stage of %d rows x %d columns does not fit a %d-byte slot", sm, k,
                  rows, t.kc, kSlotBytes);
          return MK_ERR_SCHEDULE_INVALID;
        }
        if (t.op == OP_QKV && (int)(t.u0 / (G.hd / 16)) != (int)((t.u0 + t.nunits - 1) / (G.hd / 16))) {
          set_err(err, "sm %d task %zu: a QKV task crosses a head boundary", sm, k);
          return MK_ERR_SCHEDULE_INVALID;
        }
      }
      if (t.sig_ctr >= nctr) { set_err(err, "sm %d task %zu: bad signal counter", sm, k); return MK_ERR_SCHEDULE_INVALID; }
      if (phase_of_sig[t.sig_ctr] == -1) phase_of_sig[t.sig_ctr] = pi;
      if (phase_of_sig[t.sig_ctr] != pi) {
        set_err(err, "counter %d is signalled by two phases", t.sig_ctr);
        return MK_ERR_SCHEDULE_INVALID;
      }
      n_sig[t.sig_ctr]++;
    }
  for (int pi = 0; pi < NP; ++pi) {
    std::vector<long long> id_owner(p.max_split_ids, -1);  // the first unit of the group an id belongs to
    const int op = order[pi].op;
    const int nkb = (op != OP_EMBED && op != OP_ATTN) ? (gemv_K(G, op) + kBoxCols - 1) / kBoxCols : 0;
    for (size_t u = 0; u < cover[pi].size(); ++u) {
      auto& pc = pieces[pi][u];
      bool ok = false;
      if (pc.empty()) ok = cover[pi][u] == 1;
      else if (cover[pi][u] == 0 && pc.size() >= 2 && pc.size() <= (size_t)kMaxPieces) {
        // the pieces tile [0, nkb) in K order, pieces 0..P-1 of one id with P pieces
        std::sort(pc.begin(), pc.end(), [](const Piece& a, const Piece& b) { return a.k0 < b.k0; });
        ok = pc.front().k0 == 0 && pc.back().k1 == nkb;
        const int id = split_id((uint16_t)pc[0].split);
        for (size_t k2 = 0; ok && k2 < pc.size(); ++k2) {
          const uint16_t sp = (uint16_t)pc[k2].split;
          ok = split_id(sp) == id && split_piece(sp) == (int)k2 && split_pieces(sp) == (int)pc.size() &&
               (k2 == 0 || pc[k2 - 1].k1 == pc[k2].k0) && pc[k2].u0 == pc[0].u0 && pc[k2].n == pc[0].n;
        }
        // an id names one task group (one u0) in the phase
        if (ok) {
          if (id_owner[id] < 0) id_owner[id] = pc[0].u0;
          else ok = id_owner[id] == pc[0].u0;
        }
      }
      if (!ok) {
        set_err(err, "phase op %d layer %d: unit %zu covered %d times in full and by %zu K pieces that do not "
                "pair up", order[pi].op, order[pi].layer, u, cover[pi][u], pc.size());
        return MK_ERR_SCHEDULE_INVALID;
      }
    }
  }

  // 2. every wait target is exactly the number of signals its counter gets
  for (int sm = 0; sm < nsm; ++sm)
    for (size_t k = 0; k < p.streams[sm].size(); ++k) {
      const TaskDesc& t = p.streams[sm][k];
      if (t.wait_ctr == kNoCounter) continue;
      if (t.wait_ctr >= nctr || t.wait_count != (uint32_t)n_sig[t.wait_ctr] || t.wait_count == 0) {
        set_err(err, "sm %d task %zu (op %d layer %d): waits for %u signals on counter %d, which gets %d", sm,
                k, t.op, t.layer, t.wait_count, (int)t.wait_ctr, t.wait_ctr < nctr ? n_sig[t.wait_ctr] : -1);
        return MK_ERR_SCHEDULE_INVALID;
      }
    }

  // 3. deadlock freedom: program order + counter edges must form a DAG (Kahn)
  {
    std::vector<int> first(nsm + 1, 0);
    for (int sm = 0; sm < nsm; ++sm) first[sm + 1] = first[sm] + (int)p.streams[sm].size();
    const int NT = first[nsm];
    std::vector<int> indeg(NT + nctr, 0);
    std::vector<std::vector<int>> waiters(nctr);
    for (int sm = 0; sm < nsm; ++sm)
      for (size_t k = 0; k < p.streams[sm].size(); ++k) {
        int id = first[sm] + (int)k;
        const TaskDesc& t = p.streams[sm][k];
        if (k > 0) indeg[id]++;
        if (t.wait_ctr != kNoCounter) {
          indeg[id]++;
          waiters[t.wait_ctr].push_back(id);
        }
        indeg[NT + t.sig_ctr]++;
      }
    std::vector<int> stack, sm_of(NT);
    for (int sm = 0; sm < nsm; ++sm)
      for (int id = first[sm]; id < first[sm + 1]; ++id) sm_of[id] = sm;
    for (int v = 0; v < NT + nctr; ++v)
      if (indeg[v] == 0) stack.push_back(v);
    int done = 0;
    while (!stack.empty()) {
      int v = stack.back();
      stack.pop_back();
      ++done;
      if (v < NT) {
        int sm = sm_of[v];
        const TaskDesc& t = p.streams[sm][v - first[sm]];
        if (v + 1 < first[sm + 1] && --indeg[v + 1] == 0) stack.push_back(v + 1);
        if (--indeg[NT + t.sig_ctr] == 0) stack.push_back(NT + t.sig_ctr);
      } else {
        for (int w : waiters[v - NT])
          if (--indeg[w] == 0) stack.push_back(w);
      }
    }
    if (done != NT + nctr) {
      for (int sm = 0; sm < nsm; ++sm)
        for (int id = first[sm]; id < first[sm + 1]; ++id)
          if (indeg[id] > 0) {
            const TaskDesc& t = p.streams[sm][id - first[sm]];
            set_err(err, "deadlock: sm %d task %d (op %d layer %d) can never start", sm, id - first[sm], t.op,
                    t.layer);
            return MK_ERR_SCHEDULE_INVALID;
          }
      set_err(err, "deadlock: a counter can never reach its target");
      return MK_ERR_SCHEDULE_INVALID;
    }
  }

  // 4. race freedom at phase level.  Phase A happens before phase B when every task
  // of B waits on the counter that exactly A's tasks signal; take the closure.
  {
    std::vector<int> wait_phase(NP, -2);  // -2 unset, -1 no wait, -3 mixed
    for (int sm = 0; sm < nsm; ++sm)
      for (const TaskDesc& t : p.streams[sm]) {
        int pi = phase_index(t.op, t.layer);
        int wp = t.wait_ctr == kNoCounter ? -1 : phase_of_sig[t.wait_ctr];
        if (wait_phase[pi] == -2) wait_phase[pi] = wp;
        else if (wait_phase[pi] != wp) wait_phase[pi] = -3;
      }
    std::vector<std::vector<char>> hb(NP, std::vector<char>(NP, 0));
    for (int b = 0; b < NP; ++b)
      if (wait_phase[b] >= 0) hb[wait_phase[b]][b] = 1;
    for (int k = 0; k < NP; ++k)
      for (int i = 0; i < NP; ++i)
        if (hb[i][k])
          for (int j = 0; j < NP; ++j)
            if (hb[k][j]) hb[i][j] = 1;
    for (int a = 0; a < NP; ++a)
      for (int b = a + 1; b < NP; ++b) {
        auto A = accesses(order[a].op, order[a].layer, G.L);
        auto B = accesses(order[b].op, order[b].layer, G.L);
        for (const Access& x : A)
          for (const Access& y : B)
            if (x.buf == y.buf && x.inst == y.inst && (x.write || y.write) && !hb[a][b]) {
              set_err(err, "race: phase op %d layer %d %s buffer %d and phase op %d layer %d %s it without a "
                      "counter ordering them", order[a].op, order[a].layer, x.write ? "writes" : "reads", x.buf,
                      order[b].op, order[b].layer, y.write ? "writes" : "reads");
              return MK_ERR_SCHEDULE_INVALID;
            }
      }
  }
  return MK_OK;
}

}  // namespace mk

// ---------------------------------------------------------------------------------------
// C ABI of the plan

extern "C" {

static thread_local std::string g_plan_err;
const char* mk_internal_plan_error() { return g_plan_err.c_str(); }

MK_API int mk_plan_create(const mk_model_cfg* cfg, const mk_plan_opts* opts, mk_plan_t* out) {
  if (!cfg || !out) { g_plan_err = "null argument"; return MK_ERR_INVALID_ARG; }
  mk_plan_s* p = new mk_plan_s();
  int rc = mk::build_plan(*cfg, opts, p, &g_plan_err);
  if (rc) { delete p; return rc; }
  *out = p;
  return MK_OK;
}

MK_API int mk_plan_validate(mk_plan_t plan, char* msg, size_t msg_len) {
  if (!plan) return MK_ERR_INVALID_ARG;
  std::string e;
  int rc = mk::validate_plan(*plan, &e);
  if (msg && msg_len) {
    std::snprintf(msg, msg_len, "%s", rc ? e.c_str() : "ok");
  }
  return rc;
}

MK_API int mk_plan_stats(mk_plan_t plan, mk_plan_info* o) {
  if (!plan || !o) return MK_ERR_INVALID_ARG;
  std::memset(o, 0, sizeof(*o));
  const mk::Geometry G = mk::geometry(plan->cfg);
  o->weight_bytes_min_sm = -1;
  for (const auto& s : plan->streams) {
    o->n_tasks += (int64_t)s.size();
    o->max_tasks_per_sm = std::max<int64_t>(o->max_tasks_per_sm, (int64_t)s.size());
    int64_t bytes = 0;
    for (const auto& t : s) {
      if (t.op == mk::OP_EMBED || t.op == mk::OP_ATTN) continue;
      const int K = mk::gemv_K(G, t.op);
      const int cols = std::min((int)t.k1 * mk::kBoxCols, K) - (int)t.k0 * mk::kBoxCols;
      o->n_stages += (cols + t.kc - 1) / t.kc;
      bytes += (int64_t)t.nunits * mk::rows_per_unit(t.op) * cols * 2;
    }
    o->weight_bytes_max_sm = std::max(o->weight_bytes_max_sm, bytes);
    if (o->weight_bytes_min_sm < 0 || bytes < o->weight_bytes_min_sm) o->weight_bytes_min_sm = bytes;
  }
  o->attn_slots = (int64_t)plan->num_sms * plan->attn_slots_per_sm;
  o->n_counters = mk::num_counters(G.L);
  return MK_OK;
}

MK_API int mk_plan_inject_fault(mk_plan_t plan, int32_t kind, int32_t arg) {
  if (!plan) return MK_ERR_INVALID_ARG;
  const int L = plan->cfg.n_layers;
  int layer = arg < 0 ? 0 : (arg >= L ? L - 1 : arg);
  switch (kind) {
    case MK_FAULT_DROP_WAIT: {
      for (auto& s : plan->streams)
        for (auto& t : s)
          if (t.op == mk::OP_DOWN && t.layer == layer) { t.wait_ctr = mk::kNoCounter; t.wait_count = 0; }
      return MK_OK;
    }
    case MK_FAULT_RAISE_TARGET: {
      for (auto& s : plan->streams)
        for (auto& t : s)
          if (t.op == mk::OP_LMHEAD) t.wait_count += 1;
      return MK_OK;
    }
    case MK_FAULT_REORDER: {
      // move a down task of the layer in front of a gate/up task of the same layer
      // (on the gate/up task's SM): it then waits on a task that can only run after it
      int gs = -1, gi = -1, ds = -1, di = -1;
      for (size_t s = 0; s < plan->streams.size(); ++s)
        for (size_t k = 0; k < plan->streams[s].size(); ++k) {
          const auto& t = plan->streams[s][k];
          if (t.op == mk::OP_GATEUP && t.layer == layer && gs < 0) { gs = (int)s; gi = (int)k; }
          if (t.op == mk::OP_DOWN && t.layer == layer && ds < 0) { ds = (int)s; di = (int)k; }
        }
      if (gs < 0 || ds < 0) return MK_ERR_INVALID_ARG;
      mk::TaskDesc t = plan->streams[ds][di];
      plan->streams[ds].erase(plan->streams[ds].begin() + di);
      if (ds == gs && di < gi) --gi;
      plan->streams[gs].insert(plan->streams[gs].begin() + gi, t);
      return MK_OK;
    }
    case MK_FAULT_DUP_UNIT: {
      for (auto& s : plan->streams)
        for (auto& t : s)
          if (t.op == mk::OP_OPROJ && t.layer == layer && t.nunits < 255) { t.nunits += 1; return MK_OK; }
      return MK_ERR_INVALID_ARG;
    }
    case MK_FAULT_OVERSIZE_STAGE: {
      for (auto& s : plan->streams)
        for (auto& t : s)
          if (t.op == mk::OP_LMHEAD) { t.kc = (uint16_t)(2 * mk::kSlotBytes / (t.nunits * 8)); return MK_OK; }
      return MK_ERR_INVALID_ARG;
    }
  }
  return MK_ERR_INVALID_ARG;
}

MK_API void mk_plan_destroy(mk_plan_t plan) { delete plan; }

}  // extern "C"
