// Host planner and static checker of the per-CTA task list (plain C++, no CUDA).
#pragma once
#include <string>
#include <vector>

#include "amk_internal.h"

namespace amk {

struct StageList {            // one launch of the op-per-kernel ablation
  int op = 0, layer = 0;
  std::vector<Task> tasks;
  std::vector<int> off;       // [grid + 1]
};

struct Plan {
  int grid = 0;
  int kv_chunks_max = 0;
  int kv_chunks_short = 0;
  int n_counters = 0;
  GemvGeom geom[5];
  std::vector<Task> tasks;        // persistent kernel: all CTAs' lists back to back
  std::vector<int> off;           // [grid + 1]
  std::vector<StageList> stages;  // ablation launches in order
};

// Geometry of one GEMV with rows of K elements of weight dtype `wk` (AMK_W_*); false if unsupported.
bool make_geom(int K, int wk, GemvGeom* g);

// Builds the plan. Returns AMK_OK, AMK_ERR_UNSUPPORTED or AMK_ERR_INVALID_ARG (msg says why).
int build_plan(const amk_dims& d, int grid, int kv_chunks_max, Plan* out, std::string* msg);

// Static checks (deadlock-, race- and reachability-freedom of the task list); AMK_OK or AMK_ERR_PLAN.
int check_plan(const amk_dims& d, const Plan& p, std::string* msg);

// Plants one defect (test support for the checker). Returns false if the mutation is unknown.
bool mutate_plan(Plan* p, int mutation);

// Checks the dims against what the kernels support.
int check_dims(const amk_dims& d, std::string* msg);

}  // namespace amk
