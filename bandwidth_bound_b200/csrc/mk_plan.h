// Host-side task schedule of the decode megakernel (internal header).
#pragma once
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_common.h"

struct mk_plan_s {
  mk_model_cfg cfg{};
  int num_sms = 0;
  int attn_slots_per_sm = 0;
  int max_blocks = 0;
  std::vector<std::vector<mk::TaskDesc>> streams;  // one instruction stream per SM
  std::vector<int> signalers;                      // per counter: tasks that add to it
  int max_phase_tasks = 0;                         // most tasks in one phase (scratch sizing)
  int n_lm_tasks = 0;
  int max_split_ids = 0;                           // most K-split task groups in one phase
};

namespace mk {

// Geometry shared by the builder, the validator and the launcher.
struct Geometry {
  int L, d, nq, nkv, hd, F, V, g, qdim, kvdim;
};
Geometry geometry(const mk_model_cfg& c);

int gemv_K(const Geometry& G, int op);        // input length of a GEMV op
int phase_units(const Geometry& G, int op);   // work units of one phase of op
long long unit_weight_bytes(const Geometry& G, int op);
uint16_t choose_kc(int rows, int K);          // K columns per pool stage

int check_cfg(const mk_model_cfg& c, std::string* err);
int build_plan(const mk_model_cfg& c, const mk_plan_opts* opts, mk_plan_s* out, std::string* err);
int validate_plan(const mk_plan_s& p, std::string* err);

}  // namespace mk
