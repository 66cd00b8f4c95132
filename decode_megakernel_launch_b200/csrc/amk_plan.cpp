// Host planner and static checker of the persistent kernel's task list.
//
// The checker restates, for this library's fixed task pattern, the static graph checks that
// "AutoMegaKernel: A Statically-Checked Agent Harness for Self-Retargeting Megakernel Synthesis"
// (technical summary, "The Safety Gate") runs before any launch: an acyclic producer/consumer order,
// satisfiable wait thresholds (1 <= t <= #producers), per-SM queue orders consistent with one global
// topological order, multi-producer counters joined only after every producer, each output written
// by exactly one task (no two CTAs write the same rows), every counter index valid, and the logits /
// next token reachable. A plan that fails is rejected before launch instead of hanging the GPU.
#include "amk_plan.h"

#include <algorithm>
#include <cstdio>
#include <map>
#include <set>

namespace amk {

namespace {

struct Split { int row0, nrows; };

// Rows [0, n) in units of `unit` rows, balanced over `grid` CTAs (counts differ by one unit).
std::vector<Split> split_rows(int n, int unit, int grid) {
  std::vector<Split> s(grid);
  int units = n / unit, base = units / grid, rem = units % grid, r = 0;
  for (int b = 0; b < grid; ++b) {
    int u = base + (b < rem ? 1 : 0);
    s[b] = {r * unit, u * unit};
    r += u;
  }
  return s;
}

// Stage rank inside a layer; the LM head comes after every layer.
int stage_index(int L, const Task& t) {
  switch (t.op) {
    case OP_QKV: return t.layer * 6 + 0;
    case OP_ATTN: return t.layer * 6 + 1;
    case OP_MERGE: return t.layer * 6 + 2;
    case OP_O: return t.layer * 6 + 3;
    case OP_GU: return t.layer * 6 + 4;
    case OP_DOWN: return t.layer * 6 + 5;
    case OP_LM: return L * 6 + 0;
    case OP_ARGMAX: return L * 6 + 1;
  }
  return -1;
}

int ctr_index(int layer, int kind) { return layer * CTR_PER_LAYER + kind; }

std::string fmt(const char* f, long a = 0, long b = 0, long c = 0) {
  char buf[256];
  snprintf(buf, sizeof buf, f, a, b, c);
  return buf;
}

}  // namespace

bool make_geom(int K, int wk, GemvGeom* g) {
  // Bytes per thread per row: larger groups amortise the per-slot reduction and bookkeeping over
  // more weight bytes (weight 1.0 for 32 B), smaller ones fit rows that larger ones do not divide.
  // Each candidate is scored by that efficiency times the fraction of compute warps it keeps busy.
  // A thread holds at most 32 activations: 32 B of int8, 16 B of int4 or 64 B of bf16 per row.
  const int rb = wk == AMK_W_INT4 ? K / 2 : wk == AMK_W_BF16 ? K * 2 : K;
  const int max_bytes = wk == AMK_W_INT4 ? AMK_I4_MAX_GB : wk == AMK_W_BF16 ? 64 : 32;
  const int min_bytes = wk == AMK_W_INT8 ? 2 : 4;      // bf16 and int4: at least one word per group
  if (K <= 0 || (wk == AMK_W_INT4 && (K & 1)) || rb > kSlotBytes) return false;
  bool found = false;
  double best = -1.0;
  const int gbs[] = {64, 32, 16, 8, 4, 2};
  const double eff[] = {1.0, 1.0, 0.8, 0.65, 0.5, 0.4};
  for (int i = 0; i < 6; ++i) {
    const int gb = gbs[i];
    if (gb > max_bytes || gb < min_bytes) continue;
    if (rb % gb != 0) continue;
    // groups of a row over whole warps; an int4 row's last warp may be partly filled (its idle
    // lanes count against the candidate); int8 and bf16 rows always have a whole-warp choice
    const int groups = rb / gb;
    if (wk != AMK_W_INT4 && groups % 32) continue;
    int W = (groups + 31) / 32;
    const double lane_util = double(groups) / (W * 32);
    int nr = (W + kConsumerWarps - 1) / kConsumerWarps;
    if (nr > max_bytes / gb) continue;
    int wpg = W < kConsumerWarps ? W : kConsumerWarps;
    int rp = nr == 1 ? kConsumerWarps / wpg : 1;
    double bal = nr == 1 ? double(rp * wpg) / kConsumerWarps : double(W) / (nr * kConsumerWarps);
    double score = bal * eff[i] * lane_util;
    if (score > best + 1e-9) {
      best = score;
      // rows per slot: a power of two below 8, else a multiple of 8, so every 128-row epilogue block
      // (rs * floor(128 / rs) rows) is a multiple of 8 rows: its results go out in bf16 pairs of
      // rows (SwiGLU: of two packed row pairs)
      int rs = kSlotBytes / rb;
      if (rs > 64) rs = 64;
      if (rs >= 8) rs &= ~7;
      else rs = rs >= 4 ? 4 : rs >= 2 ? 2 : 1;
      *g = GemvGeom{K, rb, gb, W, wpg, nr, rp, rs};
      found = true;
    }
  }
  return found;
}

int check_dims(const amk_dims& d, std::string* msg) {
  auto bad = [&](const char* m) { *msg = m; return AMK_ERR_UNSUPPORTED; };
  if (d.n_layers < 1 || d.d_model < 1 || d.n_q_heads < 1 || d.n_kv_heads < 1 || d.ffn < 1 || d.vocab < 1 ||
      d.max_seq < 1 || d.n_layers > kMaxLayers) {
    *msg = "dims must be positive";
    return AMK_ERR_INVALID_ARG;
  }
  if (!(d.rms_eps >= 0.0f) || !(d.rope_theta > 0.0f)) { *msg = "rope_theta must be > 0 and rms_eps >= 0"; return AMK_ERR_INVALID_ARG; }
  if (d.weight_dtype != AMK_W_INT8 && d.weight_dtype != AMK_W_BF16 && d.weight_dtype != AMK_W_INT4) {
    *msg = "weight_dtype";
    return AMK_ERR_INVALID_ARG;
  }
  if (d.head_dim != 64 && d.head_dim != 128) return bad("head_dim must be 64 or 128");
  if (d.n_q_heads % d.n_kv_heads) return bad("n_q_heads must be a multiple of n_kv_heads");
  if (d.n_q_heads / d.n_kv_heads > kMaxGroup) return bad("n_q_heads / n_kv_heads must be <= 4");
  int qd = d.n_q_heads * d.head_dim;
  for (int k : {d.d_model, d.ffn, qd})
    if (k % 64 || k > 16384) return bad("d_model, ffn and n_q_heads*head_dim must be multiples of 64, <= 16384");
  const int wk = d.weight_dtype;
  GemvGeom g;
  if (!make_geom(d.d_model, wk, &g) || !make_geom(qd, wk, &g) || !make_geom(d.ffn, wk, &g) ||
      !make_geom(d.d_model, AMK_W_BF16, &g))
    return bad("a weight row does not fit a ring slot");
  return AMK_OK;
}

int build_plan(const amk_dims& d, int grid, int kv_chunks_max, Plan* out, std::string* msg) {
  int rc = check_dims(d, msg);
  if (rc != AMK_OK) return rc;
  if (grid < 1) { *msg = "grid must be >= 1"; return AMK_ERR_INVALID_ARG; }
  Plan& p = *out;
  p = Plan();
  p.grid = grid;
  int L = d.n_layers, hd = d.head_dim, Hkv = d.n_kv_heads;
  // attention chunks per KV head; the (head, chunk) tasks go round-robin over the CTAs, so a grid
  // smaller than Hkv gives some CTAs several heads
  // at most 16 chunks per KV head by default: the merge then gathers them in one round trip
  int cmax = kv_chunks_max > 0 ? kv_chunks_max : std::min(grid / Hkv, 32);
  if (cmax < 1) cmax = 1;
  p.kv_chunks_max = cmax;
  p.kv_chunks_short = kv_chunks_max > 0 ? kv_chunks_max : std::min(grid / Hkv, 16);
  p.n_counters = L * CTR_PER_LAYER;
  const int wk = d.weight_dtype;
  make_geom(d.d_model, wk, &p.geom[0]);                           // QKV: K = d
  make_geom(d.n_q_heads * hd, wk, &p.geom[1]);                    // O:   K = Hq*hd
  make_geom(d.d_model, wk, &p.geom[2]);                           // GU:  K = d
  make_geom(d.ffn, wk, &p.geom[3]);                               // DOWN:K = ffn
  make_geom(d.d_model, d.tied_head ? AMK_W_BF16 : wk, &p.geom[4]);  // LM: its own dtype, or the bf16 table

  // results go out in pairs: QKV row pairs (RoPE), O / down rows two by two (one bf16 pair each),
  // gate/up four packed rows at a time (two SwiGLU outputs, one bf16 pair)
  int qkv_rows = (d.n_q_heads + 2 * Hkv) * hd;
  auto s_qkv = split_rows(qkv_rows, 2, grid);
  auto s_o = split_rows(d.d_model, 2, grid);
  auto s_gu = split_rows(2 * d.ffn, 4, grid);
  auto s_dn = split_rows(d.d_model, 2, grid);
  auto s_lm = split_rows(d.vocab, 1, grid);
  // remainder rows of an odd split go to the last CTA
  auto fix_tail = [&](std::vector<Split>& s, int n) {
    int covered = s.back().row0 + s.back().nrows;
    s.back().nrows += n - covered;
  };
  fix_tail(s_o, d.d_model);
  fix_tail(s_dn, d.d_model);
  fix_tail(s_lm, d.vocab);


  // Appends the tasks of one GEMV stage for CTA b: rows split into pieces of <= kMaxTaskRows
  // (even sizes for pair-wise epilogues); the first piece waits, the last signals. A CTA without
  // rows still gets one empty task so that it signals.
  auto gemv_tasks = [&](std::vector<Task>& v, int op, int layer, Split s, int wait, uint32_t mult, int sig) {
    int r = s.row0, left = s.nrows;
    bool first = true;
    do {
      int n = left < kMaxTaskRows ? left : kMaxTaskRows;
      Task t{};
      t.op = (uint16_t)op;
      t.layer = (uint16_t)layer;
      t.a = r;
      t.b = n;
      t.wait_ctr = first ? wait : -1;
      t.wait_mult = first ? mult : 0;
      left -= n;
      r += n;
      t.sig_ctr = left == 0 ? sig : -1;
      t.flags = (first ? kFirstOfStage : 0) | (left == 0 ? kLastOfStage : 0);
      v.push_back(t);
      first = false;
    } while (left > 0);
  };

  // ---- persistent kernel list ----
  p.off.assign(grid + 1, 0);
  for (int b = 0; b < grid; ++b) {
    p.off[b] = (int)p.tasks.size();
    for (int l = 0; l < L; ++l) {
      // QKV signals no counter: an attention task reads only its own KV head's q, k and v (a few
      // KB) and polls their tags, so it starts when those rows are out, not when every CTA is done
      gemv_tasks(p.tasks, OP_QKV, l, s_qkv[b], l ? ctr_index(l - 1, CTR_DOWN) : -1, l ? grid : 0, -1);
      for (int i = b; i < Hkv * cmax; i += grid) {
        Task t{};
        t.op = OP_ATTN;
        t.layer = (uint16_t)l;
        t.a = i % Hkv;
        t.b = i / Hkv;
        t.wait_ctr = -1;
        t.wait_mult = 0;
        t.sig_ctr = ctr_index(l, CTR_ATTN);   // signalled by the merging (last-arriving) chunk
        t.flags = kTagWait | (i == b ? kFirstOfStage : 0) | (i + grid >= Hkv * cmax ? kLastOfStage : 0);
        p.tasks.push_back(t);
      }
      gemv_tasks(p.tasks, OP_O, l, s_o[b], ctr_index(l, CTR_ATTN), Hkv, ctr_index(l, CTR_O));
      gemv_tasks(p.tasks, OP_GU, l, s_gu[b], ctr_index(l, CTR_O), grid, ctr_index(l, CTR_GU));
      gemv_tasks(p.tasks, OP_DOWN, l, s_dn[b], ctr_index(l, CTR_GU), grid, ctr_index(l, CTR_DOWN));
    }
    gemv_tasks(p.tasks, OP_LM, 0, s_lm[b], ctr_index(L - 1, CTR_DOWN), grid, -1);
  }
  p.off[grid] = (int)p.tasks.size();

  // ---- op-per-kernel ablation: one launch per stage, no counters ----
  auto add_stage = [&](int op, int layer, const std::vector<Split>* s) {
    StageList st;
    st.op = op;
    st.layer = layer;
    st.off.assign(grid + 1, 0);
    for (int b = 0; b < grid; ++b) {
      st.off[b] = (int)st.tasks.size();
      if (s) {
        gemv_tasks(st.tasks, op, layer, (*s)[b], -1, 0, -1);
      } else if (op == OP_ATTN) {
        for (int i = b; i < Hkv * cmax; i += grid) {
          Task t{};
          t.op = OP_ATTN; t.layer = (uint16_t)layer; t.a = i % Hkv; t.b = i / Hkv;
          t.wait_ctr = -1; t.sig_ctr = -1; t.flags = kFirstOfStage | kLastOfStage;
          st.tasks.push_back(t);
        }
      } else if (op == OP_MERGE) {
        for (int h = b; h < Hkv; h += grid) {
          Task t{};
          t.op = OP_MERGE; t.layer = (uint16_t)layer; t.a = h; t.b = 0;
          t.wait_ctr = -1; t.sig_ctr = -1; t.flags = kFirstOfStage | kLastOfStage;
          st.tasks.push_back(t);
        }
      } else if (op == OP_ARGMAX && b == 0) {
        Task t{};
        t.op = OP_ARGMAX; t.wait_ctr = -1; t.sig_ctr = -1; t.flags = kFirstOfStage | kLastOfStage;
        st.tasks.push_back(t);
      }
    }
    st.off[grid] = (int)st.tasks.size();
    p.stages.push_back(std::move(st));
  };
  for (int l = 0; l < L; ++l) {
    add_stage(OP_QKV, l, &s_qkv);
    add_stage(OP_ATTN, l, nullptr);
    add_stage(OP_MERGE, l, nullptr);
    add_stage(OP_O, l, &s_o);
    add_stage(OP_GU, l, &s_gu);
    add_stage(OP_DOWN, l, &s_dn);
  }
  add_stage(OP_LM, 0, &s_lm);
  add_stage(OP_ARGMAX, 0, nullptr);
  return AMK_OK;
}

int check_plan(const amk_dims& d, const Plan& p, std::string* msg) {
  auto fail = [&](const std::string& m) { *msg = m; return AMK_ERR_PLAN; };
  int L = d.n_layers, grid = p.grid, Hkv = d.n_kv_heads;
  if ((int)p.off.size() != grid + 1 || p.off[0] != 0 || p.off[grid] != (int)p.tasks.size())
    return fail("task offsets do not cover the task list");
  const int nctr = p.n_counters;
  // producers per counter per step; which stage produces it
  std::vector<int> producers(nctr, 0), prod_stage(nctr, -1);
  std::vector<std::vector<int>> attn_heads(L);  // chunk-0 tasks per (layer) by head
  for (int l = 0; l < L; ++l) attn_heads[l].assign(Hkv, 0);
  for (int b = 0; b < grid; ++b) {
    int prev = -1;
    std::set<int> signalled;
    for (int i = p.off[b]; i < p.off[b + 1]; ++i) {
      const Task& t = p.tasks[i];
      int st = stage_index(L, t);
      if (st < 0 || t.layer >= L) return fail(fmt("CTA %ld task %ld: unknown op or layer", b, i - p.off[b]));
      if (st < prev) return fail(fmt("CTA %ld: task %ld breaks the global stage order", b, i - p.off[b]));
      prev = st;
      if (t.wait_ctr < -1 || t.wait_ctr >= nctr || t.sig_ctr < -1 || t.sig_ctr >= nctr)
        return fail(fmt("CTA %ld task %ld: counter index out of range", b, i - p.off[b]));
      if (t.sig_ctr >= 0) {
        if (signalled.count(t.sig_ctr) && t.op != OP_ATTN)
          return fail(fmt("CTA %ld signals counter %ld twice per step", b, t.sig_ctr));
        signalled.insert(t.sig_ctr);
        if (t.op == OP_ATTN) {
          if (t.a < 0 || t.a >= Hkv || t.b < 0 || t.b >= p.kv_chunks_max)
            return fail(fmt("CTA %ld: attention task out of range", b));
          if (t.b == 0) attn_heads[t.layer][t.a]++;
        } else {
          producers[t.sig_ctr]++;
        }
        int& ps = prod_stage[t.sig_ctr];
        if (ps >= 0 && ps != st) return fail(fmt("counter %ld is signalled from two stages", t.sig_ctr));
        ps = st;
      }
    }
  }
  // attention counters: one signal per KV head (the merging chunk of that head)
  for (int l = 0; l < L; ++l)
    for (int h = 0; h < Hkv; ++h) {
      if (attn_heads[l][h] != 1) return fail(fmt("layer %ld KV head %ld has %ld chunk-0 attention tasks", l, h, attn_heads[l][h]));
      producers[ctr_index(l, CTR_ATTN)]++;
    }
  // waits: backwards only, thresholds satisfiable and joining every producer
  for (int b = 0; b < grid; ++b)
    for (int i = p.off[b]; i < p.off[b + 1]; ++i) {
      const Task& t = p.tasks[i];
      if (t.wait_ctr < 0) continue;
      int st = stage_index(L, t);
      int ps = prod_stage[t.wait_ctr];
      if (ps < 0) return fail(fmt("CTA %ld waits on counter %ld that nothing signals", b, t.wait_ctr));
      if (ps >= st) return fail(fmt("CTA %ld waits on counter %ld produced at or after its own stage", b, t.wait_ctr));
      if (t.wait_mult < 1 || (int)t.wait_mult > producers[t.wait_ctr])
        return fail(fmt("counter %ld: threshold %ld exceeds its %ld producers", t.wait_ctr, t.wait_mult, producers[t.wait_ctr]));
      if ((int)t.wait_mult != producers[t.wait_ctr])
        return fail(fmt("counter %ld: threshold %ld does not join all %ld producers", t.wait_ctr, t.wait_mult, producers[t.wait_ctr]));
    }
  // every stage after the first waits on its predecessor: on its counter, or (attention, whose
  // inputs are one KV head's q, k and v) on the tags of the same layer's QKV output
  for (int b = 0; b < grid; ++b)
    for (int i = p.off[b]; i < p.off[b + 1]; ++i) {
      const Task& t = p.tasks[i];
      if (t.op == OP_ATTN) {
        if (!(t.flags & kTagWait) || t.wait_ctr != -1)
          return fail(fmt("CTA %ld task %ld: an attention task must poll its inputs' tags", b, i - p.off[b]));
        continue;
      }
      if (t.flags & kTagWait) return fail(fmt("CTA %ld task %ld: only attention polls tags", b, i - p.off[b]));
      if (!(t.flags & kFirstOfStage) || (t.op == OP_QKV && t.layer == 0)) continue;
      int want = t.op == OP_QKV ? ctr_index(t.layer - 1, CTR_DOWN)
               : t.op == OP_O ? ctr_index(t.layer, CTR_ATTN)
               : t.op == OP_GU ? ctr_index(t.layer, CTR_O)
               : t.op == OP_DOWN ? ctr_index(t.layer, CTR_GU)
               : ctr_index(L - 1, CTR_DOWN);
      if (t.wait_ctr != want) return fail(fmt("CTA %ld task %ld does not wait for its input stage", b, i - p.off[b]));
    }
  // outputs: each GEMV stage's rows written exactly once over all CTAs
  int qkv_rows = (d.n_q_heads + 2 * Hkv) * d.head_dim;
  std::map<std::pair<int, int>, std::vector<std::pair<int, int>>> rows;
  for (const Task& t : p.tasks)
    if (t.op != OP_ATTN) rows[{t.op, t.layer}].push_back({t.a, t.b});
  auto need = [&](int op) {
    return op == OP_QKV ? qkv_rows : op == OP_O || op == OP_DOWN ? d.d_model : op == OP_GU ? 2 * d.ffn : d.vocab;
  };
  for (int l = 0; l < L; ++l)
    for (int op : {OP_QKV, OP_O, OP_GU, OP_DOWN}) {
      auto it = rows.find({op, l});
      if (it == rows.end()) return fail(fmt("layer %ld stage %ld has no tasks", l, op));
    }
  if (!rows.count({OP_LM, 0})) return fail("no LM-head task: logits and next token unreachable");
  for (auto& kv : rows) {
    auto v = kv.second;
    std::sort(v.begin(), v.end());
    int r = 0;
    for (auto& s : v) {
      if (s.second == 0) continue;
      if (s.first != r) return fail(fmt("stage %ld layer %ld: rows overlap or leave a gap at %ld", kv.first.first, kv.first.second, r));
      r += s.second;
    }
    if (r != need(kv.first.first)) return fail(fmt("stage %ld layer %ld covers %ld rows", kv.first.first, kv.first.second, r));
  }
  // pair-wise epilogues: QKV, O and down rows in pairs, gate/up rows in fours
  for (const Task& t : p.tasks) {
    const int unit = t.op == OP_GU ? 4 : (t.op == OP_QKV || t.op == OP_O || t.op == OP_DOWN) ? 2 : 1;
    if ((t.a % unit) || (t.b % unit)) return fail(fmt("stage %ld: task rows %ld + %ld split a row pair", t.op, t.a, t.b));
  }
  *msg = "ok";
  return AMK_OK;
}

bool mutate_plan(Plan* p, int mutation) {
  auto find = [&](int op, int layer) -> Task* {
    for (auto& t : p->tasks)
      if (t.op == op && t.layer == layer && t.sig_ctr >= 0) return &t;
    return nullptr;
  };
  switch (mutation) {
    case 0: return true;
    case 1: { Task* t = find(OP_GU, 0); if (!t) return false; t->sig_ctr = -1; return true; }      // dropped signal
    case 2: { for (auto& t : p->tasks) if (t.wait_ctr >= 0) { t.wait_mult += 1; return true; } return false; }
    case 3: {                                                                                      // reorder one queue
      int b = p->grid - 1;
      std::swap(p->tasks[p->off[b]], p->tasks[p->off[b] + 2]);
      return true;
    }
    case 4: { for (auto& t : p->tasks) if (t.op == OP_O && t.wait_ctr >= 0) { t.wait_ctr += 2; return true; } return false; }
    case 5: {                                                                                      // lose a producer
      for (size_t i = 0; i < p->tasks.size(); ++i)
        if (p->tasks[i].op == OP_DOWN && p->tasks[i].b > 0) {
          p->tasks.erase(p->tasks.begin() + i);
          for (auto& o : p->off) if (o > (int)i) --o;
          return true;
        }
      return false;
    }
  }
  return false;
}

}  // namespace amk
