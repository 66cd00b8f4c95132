// amk_decode_step_noalloc: the decode step for callers that cannot allocate device memory.
//
// Some callers can't call cudaMalloc: a plugin running inside a host framework whose memory pool owns
// all of the device memory (an outside cudaMalloc either fails near the pool's limit or is forbidden
// by the host's policy), or a latency-critical loop where cudaMalloc / cudaFree may synchronize the
// whole device. amk_create allocates its own device state (task list, scratch vectors, counters,
// RoPE table), so those callers cannot use it. This entry point keeps the same state in one
// file-scope static device array instead and launches the same persistent kernel as
// amk_decode_step; the caller still passes every input and output buffer.
//
// The array is fixed at kNoAllocScratchBytes (4 MiB) and stays resident on every GPU that loads the
// library until the process exits. Set-up: the first call on a device (with that device current)
// looks up the array's device address with cudaGetSymbolAddress and sets the kernel's
// shared-memory attribute; make that first call before any stream capture. Every call shares the
// array and it keeps the last call's contents: each call clears the counters, tickets and status
// words that must start at zero, and re-uploads the task list / RoPE table / layer pointers when the
// dims, weights or device differ from the previous call. Calls whose launches overlap on the GPU
// (different streams, no ordering between them) race on the array.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "amk_internal.h"
#include "amk_plan.h"

namespace amk {
cudaError_t prepare_kernel_attributes();
cudaError_t occupancy(int* blocks_per_sm);
cudaError_t launch_decode(const Params& p, cudaStream_t stream, bool cooperative);
}  // namespace amk

using namespace amk;

namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;   // the stated maximum
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct DeviceSlot {
  bool ready = false;
  unsigned char* base = nullptr;   // device address of g_noalloc_scratch on this device
  int sms = 0;
  int per_sm = 0;
  // what the array currently holds
  bool loaded = false;
  amk_dims dims{};
  std::vector<const void*> ptrs;   // weight / cache pointers the uploaded LayerPtrs came from
  Params base_params{};
  size_t zero_off = 0, zero_bytes = 0;
  uint32_t tag_epoch = 0;          // tag epoch of the last call
};

std::mutex g_mu;
DeviceSlot g_dev[kMaxDevices];

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::vector<const void*> pointer_list(const amk_dims& d, const amk_weights& w) {
  std::vector<const void*> v = {w.embed, w.final_norm, w.lm_head, w.slm, w.k_cache, w.v_cache};
  const bool i8 = d.weight_dtype != AMK_W_BF16;   // quantised weights carry row scales
  for (int l = 0; l < d.n_layers; ++l) {
    v.insert(v.end(), {w.attn_norm[l], w.ffn_norm[l], w.wqkv[l], w.wo[l], w.wgu[l], w.wdown[l]});
    if (i8) v.insert(v.end(), {w.sqkv[l], w.so[l], w.sgu[l], w.sdown[l]});
  }
  return v;
}

bool same_dims(const amk_dims& a, const amk_dims& b) { return std::memcmp(&a, &b, sizeof(amk_dims)) == 0; }

}  // namespace

extern "C" int amk_decode_step_noalloc(const amk_dims* dims, const amk_weights* w, int token_id, int pos,
                                       float* logits_out, int* next_token_out, void* stream) {
  if (!dims || !w || !next_token_out) return AMK_ERR_INVALID_ARG;
  const amk_dims& d = *dims;
  std::string msg;
  int rc = check_dims(d, &msg);
  if (rc) return rc;
  if (pos < 0 || pos >= d.max_seq || token_id < -1 || token_id >= d.vocab) return AMK_ERR_INVALID_ARG;
  const int L = d.n_layers;
  const bool i8 = d.weight_dtype != AMK_W_BF16;   // quantised weights carry row scales
  if (!aligned16(w->embed) || !aligned16(w->final_norm) || !aligned16(w->k_cache) || !aligned16(w->v_cache) ||
      !w->attn_norm || !w->ffn_norm || !w->wqkv || !w->wo || !w->wgu || !w->wdown)
    return AMK_ERR_INVALID_ARG;
  if (!d.tied_head && !aligned16(w->lm_head)) return AMK_ERR_INVALID_ARG;
  if (i8 && (!w->sqkv || !w->so || !w->sgu || !w->sdown || (!d.tied_head && !w->slm))) return AMK_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    if (!aligned16(w->attn_norm[l]) || !aligned16(w->ffn_norm[l]) || !aligned16(w->wqkv[l]) || !aligned16(w->wo[l]) ||
        !aligned16(w->wgu[l]) || !aligned16(w->wdown[l]))
      return AMK_ERR_INVALID_ARG;
    if (i8 && (!w->sqkv[l] || !w->so[l] || !w->sgu[l] || !w->sdown[l])) return AMK_ERR_INVALID_ARG;
  }

  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return AMK_ERR_CUDA;
  DeviceSlot& S = g_dev[dev];
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // ---- once per device: the array's device address, kernel attributes, co-residency ----
  if (!S.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return AMK_ERR_CUDA;
    int coop = 0;
    if (cudaDeviceGetAttribute(&S.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return AMK_ERR_CUDA;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (prepare_kernel_attributes() != cudaSuccess || occupancy(&S.per_sm) != cudaSuccess) return AMK_ERR_CUDA;
    if (!coop || S.per_sm < 1) return AMK_ERR_NOT_RESIDENT;
    S.base = static_cast<unsigned char*>(ptr);
    S.ready = true;
  }

  // ---- (re)load the plan, layer pointers and RoPE table when the model differs ----
  std::vector<const void*> ptrs = pointer_list(d, *w);
  if (!S.loaded || !same_dims(S.dims, d) || S.ptrs != ptrs) {
    // a reload copies from pageable host memory, which stream capture does not allow: refuse it
    // before enqueuing anything (a capture would be invalidated)
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return AMK_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return AMK_ERR_INVALID_ARG;
    S.loaded = false;
    const int grid = S.sms;
    Plan pl;
    if ((rc = build_plan(d, grid, 0, &pl, &msg)) != AMK_OK) return rc;
    if ((rc = check_plan(d, pl, &msg)) != AMK_OK) return rc;
    const int G = d.n_q_heads / d.n_kv_heads, half = d.head_dim / 2;
    // layout of the array
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
    const size_t o_tasks = take(pl.tasks.size() * sizeof(Task));
    const size_t o_off = take(pl.off.size() * sizeof(int));
    const size_t o_layers = take((size_t)L * sizeof(LayerPtrs));
    const size_t o_rope = take((size_t)d.max_seq * half * 2 * sizeof(float));
    const size_t tagged_begin = off;                      // tagged vectors: zeroed on every reload
    const size_t o_x = take((size_t)d.d_model / 2 * 8);
    const size_t o_xres = take((size_t)d.d_model * 4);
    const size_t o_qkv = take((size_t)(d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim * 8);
    const size_t o_ao = take((size_t)d.n_q_heads * d.head_dim / 2 * 8);
    const size_t o_act = take((size_t)d.ffn / 2 * 8);
    const size_t o_part = take((size_t)d.n_kv_heads * pl.kv_chunks_max * G * (d.head_dim + 2) * 8);
    const size_t o_am = take((size_t)grid * 16);
    const size_t zero_begin = off;                        // everything below must start at zero
    const size_t o_ctr = take((size_t)pl.n_counters * 4);
    const size_t o_tix = take((size_t)L * d.n_kv_heads * 4);
    const size_t o_amt = take(4);
    const size_t o_abort = take(4);
    const size_t o_status = take(4);
    const size_t total = off;
    if (total > kNoAllocScratchBytes) return AMK_ERR_SCRATCH_LIMIT;

    std::vector<LayerPtrs> lp(L);
    for (int l = 0; l < L; ++l) {
      lp[l].wqkv = w->wqkv[l]; lp[l].wo = w->wo[l]; lp[l].wgu = w->wgu[l]; lp[l].wdown = w->wdown[l];
      lp[l].sqkv = i8 ? static_cast<const uint16_t*>(w->sqkv[l]) : nullptr;
      lp[l].so = i8 ? static_cast<const uint16_t*>(w->so[l]) : nullptr;
      lp[l].sgu = i8 ? static_cast<const uint16_t*>(w->sgu[l]) : nullptr;
      lp[l].sdown = i8 ? static_cast<const uint16_t*>(w->sdown[l]) : nullptr;
      lp[l].attn_norm = static_cast<const uint16_t*>(w->attn_norm[l]);
      lp[l].ffn_norm = static_cast<const uint16_t*>(w->ffn_norm[l]);
    }
    std::vector<float> rope((size_t)d.max_seq * half * 2);
    for (int ps = 0; ps < d.max_seq; ++ps)
      for (int i = 0; i < half; ++i) {
        const double a = (double)ps * std::pow((double)d.rope_theta, -2.0 * i / d.head_dim);
        rope[((size_t)ps * half + i) * 2] = (float)std::cos(a);
        rope[((size_t)ps * half + i) * 2 + 1] = (float)std::sin(a);
      }
    unsigned char* B = S.base;
    auto put = [&](size_t o, const void* src, size_t bytes) {
      return bytes == 0 || cudaMemcpyAsync(B + o, src, bytes, cudaMemcpyHostToDevice, st) == cudaSuccess;
    };
    if (!put(o_tasks, pl.tasks.data(), pl.tasks.size() * sizeof(Task)) ||
        !put(o_off, pl.off.data(), pl.off.size() * sizeof(int)) ||
        !put(o_layers, lp.data(), lp.size() * sizeof(LayerPtrs)) || !put(o_rope, rope.data(), rope.size() * 4))
      return AMK_ERR_CUDA;
    // tag 0 never matches (tag epochs start at 1): no value left by another model passes a check
    if (cudaMemsetAsync(B + tagged_begin, 0, zero_begin - tagged_begin, st) != cudaSuccess) return AMK_ERR_CUDA;
    S.tag_epoch = 0;

    Params& p = S.base_params;
    p = Params{};
    p.L = L; p.d = d.d_model; p.Hq = d.n_q_heads; p.Hkv = d.n_kv_heads; p.hd = d.head_dim; p.ffn = d.ffn;
    p.V = d.vocab; p.max_seq = d.max_seq; p.eps = d.rms_eps; p.wdtype = d.weight_dtype; p.tied = d.tied_head;
    p.grid = grid;
    p.layers = reinterpret_cast<const LayerPtrs*>(B + o_layers);
    p.embed = static_cast<const uint16_t*>(w->embed);
    p.final_norm = static_cast<const uint16_t*>(w->final_norm);
    p.lm_w = d.tied_head ? w->embed : w->lm_head;
    p.lm_s = (!d.tied_head && i8) ? static_cast<const uint16_t*>(w->slm) : nullptr;
    p.kcache = static_cast<uint16_t*>(w->k_cache);
    p.vcache = static_cast<uint16_t*>(w->v_cache);
    if (encode_kv_maps(p) != AMK_OK) return AMK_ERR_CUDA;
    p.rope = reinterpret_cast<const float*>(B + o_rope);
    p.x = reinterpret_cast<uint64_t*>(B + o_x);
    p.xres = reinterpret_cast<float*>(B + o_xres);
    p.qkv = reinterpret_cast<uint64_t*>(B + o_qkv);
    p.attn_out = reinterpret_cast<uint64_t*>(B + o_ao);
    p.act = reinterpret_cast<uint64_t*>(B + o_act);
    p.attn_part = reinterpret_cast<uint64_t*>(B + o_part);
    p.am = reinterpret_cast<uint64_t*>(B + o_am);
    p.ctr = reinterpret_cast<uint32_t*>(B + o_ctr);
    p.attn_ticket = reinterpret_cast<uint32_t*>(B + o_tix);
    p.am_ticket = reinterpret_cast<uint32_t*>(B + o_amt);
    p.abort_flag = reinterpret_cast<uint32_t*>(B + o_abort);
    p.status = reinterpret_cast<volatile uint32_t*>(B + o_status);
    p.trace = nullptr;
    p.max_tasks_per_cta = 0;
    p.tasks = reinterpret_cast<const Task*>(B + o_tasks);
    p.task_off = reinterpret_cast<const int*>(B + o_off);
    for (int i = 0; i < 5; ++i) p.geom[i] = pl.geom[i];
    p.kv_block = 64;
    p.kv_chunks_max = pl.kv_chunks_max;
    p.kv_chunks_short = pl.kv_chunks_short;
    p.timeout_ns = 2000ull * 1000000ull;
    S.zero_off = zero_begin;
    S.zero_bytes = total - zero_begin;
    S.dims = d;
    S.ptrs = std::move(ptrs);
    S.loaded = true;
  }

  // ---- per call: zero the counters / tickets / status, then one persistent launch ----
  if (cudaMemsetAsync(S.base + S.zero_off, 0, S.zero_bytes, st) != cudaSuccess) return AMK_ERR_CUDA;
  // counters restart from zero each call, so their targets use epoch 1; the tags use a running
  // epoch, so no value left in the array by an earlier call passes a check
  Params p = S.base_params;
  p.epoch = 1;
  S.tag_epoch = S.tag_epoch + 1 == 0 ? 1 : S.tag_epoch + 1;
  p.tag_epoch = S.tag_epoch;
  p.token = token_id;
  p.pos = pos;
  p.logits = logits_out;
  p.next_token = next_token_out;
  p.sync = 1;
  return launch_decode(p, st, true) == cudaSuccess ? AMK_OK : AMK_ERR_CUDA;
}
