// Host side of the libamk C ABI (see include/amk.h for the contract of every call).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "amk_internal.h"
#include "amk_plan.h"

namespace amk {
cudaError_t prepare_kernel_attributes();
cudaError_t occupancy(int* blocks_per_sm);
cudaError_t launch_decode(const Params& p, cudaStream_t stream, bool cooperative);
cudaError_t launch_pack(int role, int hd, int ffn, const void* src, int src_dtype, int rows, int cols, int dst_dtype,
                        void* dst, void* scales, cudaStream_t stream);
}  // namespace amk

using namespace amk;

namespace {
thread_local std::string g_cuda_error;
}

namespace amk {

int encode_kv_maps(Params& p) {
  using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeTiled encode = nullptr;
  if (!encode) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !f) {
      g_cuda_error = "cuTensorMapEncodeTiled: not available from the driver";
      return AMK_ERR_CUDA;
    }
    encode = reinterpret_cast<EncodeTiled>(f);
  }
  // [L * Hkv * max_seq rows][hd] bf16; boxes of 64 elements (128 bytes) by 64 or 16 rows, swizzled
  // so that the rows of an 8-row tile fall in distinct bank groups; rows past the end read as zero
  const cuuint64_t dims[2] = {(cuuint64_t)p.hd, (cuuint64_t)p.L * p.Hkv * p.max_seq};
  const cuuint64_t strides[1] = {(cuuint64_t)p.hd * 2};
  const cuuint32_t unit[2] = {1, 1};
  for (int b = 0; b < 2; ++b) {
    const cuuint32_t box[2] = {64, b ? 16u : 64u};
    for (int i = 0; i < 2; ++i) {
      const CUresult r = encode(i ? &p.vmap[b] : &p.kmap[b], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, i ? p.vcache : p.kcache,
                                dims, strides, box, unit, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) {
        g_cuda_error = "cuTensorMapEncodeTiled refused the KV cache layout (error " + std::to_string((int)r) + ")";
        return AMK_ERR_CUDA;
      }
    }
  }
  return AMK_OK;
}

}  // namespace amk

namespace {

int cuda_fail(cudaError_t e, const char* what) {
  g_cuda_error = std::string(what) + ": " + cudaGetErrorString(e);
  return AMK_ERR_CUDA;
}
#define AMK_CUDA(call)                                  \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceStage {
  int op, layer;
  Task* tasks;
  int* off;
};

}  // namespace

struct amk_handle {
  amk_dims dims{};
  amk_options opt{};
  Plan plan;
  int device = 0;
  Params base{};               // launch parameters except the per-launch fields
  std::vector<void*> allocs;   // device allocations owned by the handle
  uint32_t* status_host = nullptr;
  uint32_t epoch = 0;
  std::vector<DeviceStage> stages;
  int max_tasks_per_cta = 0;

  ~amk_handle() {
    cudaSetDevice(device);
    cudaDeviceSynchronize();
    for (void* p : allocs) cudaFree(p);
    if (status_host) cudaFreeHost(status_host);
  }
  template <class T>
  int alloc(T** out, size_t count, bool zero = true) {
    void* p = nullptr;
    size_t bytes = count * sizeof(T);
    if (bytes == 0) bytes = 16;
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return e == cudaErrorMemoryAllocation ? AMK_ERR_NO_MEMORY : cuda_fail(e, "cudaMalloc");
    allocs.push_back(p);
    if (zero) {
      e = cudaMemset(p, 0, bytes);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemset");
    }
    *out = static_cast<T*>(p);
    return AMK_OK;
  }
  template <class T>
  int upload(T** out, const std::vector<T>& v) {
    int rc = alloc(out, v.size(), false);
    if (rc) return rc;
    if (!v.empty()) AMK_CUDA(cudaMemcpy(*out, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice));
    return AMK_OK;
  }
};

extern "C" {

const char* amk_last_cuda_error(void) { return g_cuda_error.c_str(); }

size_t amk_packed_bytes(int rows, int cols, int dst_dtype) {
  if (rows < 0 || cols < 0 || (dst_dtype != AMK_W_INT8 && dst_dtype != AMK_W_BF16 && dst_dtype != AMK_W_INT4))
    return 0;
  if (dst_dtype == AMK_W_INT4) return (cols & 1) ? 0 : (size_t)rows * (size_t)cols / 2;
  return (size_t)rows * (size_t)cols * (dst_dtype == AMK_W_INT8 ? 1 : 2);
}

int amk_packed_row_source(int role, const amk_dims* dims, int rows, int packed_row) {
  if (packed_row < 0 || packed_row >= rows || role < AMK_ROLE_PLAIN || role > AMK_ROLE_LM_HEAD) return -1;
  if ((role == AMK_ROLE_QKV || role == AMK_ROLE_GATE_UP) && !dims) return -1;
  int hd = dims ? dims->head_dim : 1, ffn = dims ? dims->ffn : 0;
  if (role == AMK_ROLE_QKV && (hd <= 0 || rows % hd)) return -1;
  if (role == AMK_ROLE_GATE_UP && rows != 2 * ffn) return -1;
  return packed_row_source(role, hd, ffn, packed_row);
}

int amk_pack_weight(int role, const amk_dims* dims, const void* src, int src_dtype, int rows, int cols, int dst_dtype,
                    void* packed_out, void* scales_out, void* stream) {
  if (!src || !packed_out || rows < 1 || cols < 1) return AMK_ERR_INVALID_ARG;
  if (src_dtype != AMK_SRC_F32 && src_dtype != AMK_SRC_BF16) return AMK_ERR_INVALID_ARG;
  if (dst_dtype != AMK_W_INT8 && dst_dtype != AMK_W_BF16 && dst_dtype != AMK_W_INT4) return AMK_ERR_INVALID_ARG;
  if (dst_dtype != AMK_W_BF16 && !scales_out) return AMK_ERR_INVALID_ARG;
  if (dst_dtype == AMK_W_INT4 && (cols & 1)) return AMK_ERR_INVALID_ARG;
  if (role < AMK_ROLE_PLAIN || role > AMK_ROLE_LM_HEAD) return AMK_ERR_INVALID_ARG;
  int hd = 1, ffn = 0;
  if (role != AMK_ROLE_PLAIN) {
    if (!dims) return AMK_ERR_INVALID_ARG;
    hd = dims->head_dim;
    ffn = dims->ffn;
    int d = dims->d_model, qd = dims->n_q_heads * dims->head_dim;
    int want_r = 0, want_c = 0;
    switch (role) {
      case AMK_ROLE_QKV: want_r = (dims->n_q_heads + 2 * dims->n_kv_heads) * hd; want_c = d; break;
      case AMK_ROLE_O: want_r = d; want_c = qd; break;
      case AMK_ROLE_GATE_UP: want_r = 2 * ffn; want_c = d; break;
      case AMK_ROLE_DOWN: want_r = d; want_c = ffn; break;
      case AMK_ROLE_LM_HEAD: want_r = dims->vocab; want_c = d; break;
    }
    if (rows != want_r || cols != want_c) return AMK_ERR_INVALID_ARG;
  }
  cudaError_t e = launch_pack(role, hd, ffn, src, src_dtype, rows, cols, dst_dtype, packed_out, scales_out,
                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AMK_OK : cuda_fail(e, "pack_kernel");
}

uint64_t amk_step_bytes(const amk_dims* d, int pos) {
  if (!d || pos < 0) return 0;
  const uint64_t L = d->n_layers, dm = d->d_model, hd = d->head_dim, hq = d->n_q_heads, hkv = d->n_kv_heads,
                 ffn = d->ffn, V = d->vocab;
  const int wd = d->weight_dtype;
  auto wb = [wd](uint64_t elems) { return wd == AMK_W_INT4 ? elems / 2 : wd == AMK_W_BF16 ? elems * 2 : elems; };
  const uint64_t sc = wd == AMK_W_BF16 ? 0 : 2;   // one bf16 scale per row of quantised weights
  const uint64_t qkv_rows = (hq + 2 * hkv) * hd;
  uint64_t per_layer = wb(qkv_rows * dm) + qkv_rows * sc             // QKV
                       + wb(dm * hq * hd) + dm * sc                  // O
                       + wb(2 * ffn * dm) + 2 * ffn * sc             // gate + up
                       + wb(dm * ffn) + dm * sc;                     // down
  uint64_t head = d->tied_head ? V * dm * 2 : wb(V * dm) + V * sc;
  uint64_t gains = (2 * L + 1) * dm * 2;
  uint64_t kv = 2ull * L * hkv * (uint64_t)(pos + 1) * hd * 2;
  return L * per_layer + head + dm * 2 /*embedding row*/ + gains + kv;
}

int amk_plan_check(const amk_dims* dims, int grid, int mutation, char* msg, int msg_len) {
  if (!dims) return AMK_ERR_INVALID_ARG;
  Plan p;
  std::string m;
  int rc = build_plan(*dims, grid, 0, &p, &m);
  if (rc == AMK_OK) {
    if (!mutate_plan(&p, mutation)) {
      m = "unknown mutation";
      rc = AMK_ERR_INVALID_ARG;
    } else {
      rc = check_plan(*dims, p, &m);
    }
  }
  if (msg && msg_len > 0) {
    strncpy(msg, m.c_str(), msg_len - 1);
    msg[msg_len - 1] = 0;
  }
  return rc;
}

int amk_create(const amk_dims* dims, const amk_weights* w, const amk_options* options, amk_handle** out) {
  if (!out) return AMK_ERR_INVALID_ARG;
  *out = nullptr;
  if (!dims || !w) return AMK_ERR_INVALID_ARG;
  const amk_dims& d = *dims;
  std::string msg;
  int rc = check_dims(d, &msg);
  if (rc) {
    g_cuda_error = msg;
    return rc;
  }
  const int L = d.n_layers;
  const bool i8 = d.weight_dtype != AMK_W_BF16;   // quantised (int8 or int4) weights carry row scales
  // pointer checks
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

  amk_handle* h = new amk_handle();
  auto fail = [&](int code) {
    delete h;
    return code;
  };
  h->dims = d;
  if (options) h->opt = *options;
  if (cudaGetDevice(&h->device) != cudaSuccess) return fail(cuda_fail(cudaGetLastError(), "cudaGetDevice"));
  int sms = 0, coop = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device);
  if (e != cudaSuccess) return fail(cuda_fail(e, "cudaDeviceGetAttribute"));
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, h->device);
  int grid = h->opt.grid > 0 ? h->opt.grid : sms;
  if ((e = prepare_kernel_attributes()) != cudaSuccess) return fail(cuda_fail(e, "cudaFuncSetAttribute"));
  int per_sm = 0;
  if ((e = occupancy(&per_sm)) != cudaSuccess) return fail(cuda_fail(e, "occupancy"));
  if (!coop || per_sm < 1 || grid > per_sm * sms) return fail(AMK_ERR_NOT_RESIDENT);

  rc = build_plan(d, grid, h->opt.max_kv_chunks, &h->plan, &msg);
  if (rc) {
    g_cuda_error = msg;
    return fail(rc);
  }
  rc = check_plan(d, h->plan, &msg);
  if (rc) {
    g_cuda_error = msg;
    return fail(rc);
  }
  if (h->opt.test_drop_signal > 0) {
    // test support: remove one signal AFTER the static check, so the device waits must expire
    int k = h->opt.test_drop_signal - 1;
    for (auto& t : h->plan.tasks)
      if (t.sig_ctr >= 0 && k-- == 0) { t.sig_ctr = -1; break; }
  }
  const Plan& pl = h->plan;
  for (int b = 0; b < grid; ++b) h->max_tasks_per_cta = std::max(h->max_tasks_per_cta, pl.off[b + 1] - pl.off[b]);

  Params& p = h->base;
  p.L = L; p.d = d.d_model; p.Hq = d.n_q_heads; p.Hkv = d.n_kv_heads; p.hd = d.head_dim; p.ffn = d.ffn;
  p.V = d.vocab; p.max_seq = d.max_seq; p.eps = d.rms_eps; p.wdtype = d.weight_dtype; p.tied = d.tied_head;
  p.grid = grid;
  p.embed = static_cast<const uint16_t*>(w->embed);
  p.final_norm = static_cast<const uint16_t*>(w->final_norm);
  p.lm_w = d.tied_head ? w->embed : w->lm_head;
  p.lm_s = (!d.tied_head && i8) ? static_cast<const uint16_t*>(w->slm) : nullptr;
  p.kcache = static_cast<uint16_t*>(w->k_cache);
  p.vcache = static_cast<uint16_t*>(w->v_cache);
  if ((rc = encode_kv_maps(p))) return fail(rc);
  for (int i = 0; i < 5; ++i) p.geom[i] = pl.geom[i];
  p.kv_block = h->opt.kv_block > 0 ? h->opt.kv_block : 64;
  p.kv_chunks_max = pl.kv_chunks_max;
  p.kv_chunks_short = pl.kv_chunks_short;
  p.timeout_ns = (unsigned long long)(h->opt.timeout_ms > 0 ? h->opt.timeout_ms : 2000) * 1000000ull;
  p.max_tasks_per_cta = h->max_tasks_per_cta;

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
  LayerPtrs* lp_d;
  if ((rc = h->upload(&lp_d, lp))) return fail(rc);
  p.layers = lp_d;

  // RoPE table: angles pos * theta^(-2i/hd) in float64, stored as fp32 (cos, sin)
  const int half = d.head_dim / 2;
  std::vector<float> rope((size_t)d.max_seq * half * 2);
  for (int ps = 0; ps < d.max_seq; ++ps)
    for (int i = 0; i < half; ++i) {
      const double inv = std::pow((double)d.rope_theta, -2.0 * i / d.head_dim);
      const double a = (double)ps * inv;
      rope[((size_t)ps * half + i) * 2] = (float)std::cos(a);
      rope[((size_t)ps * half + i) * 2 + 1] = (float)std::sin(a);
    }
  float* rope_d;
  if ((rc = h->upload(&rope_d, rope))) return fail(rc);
  p.rope = rope_d;

  const int G = d.n_q_heads / d.n_kv_heads;
  // tagged vectors start zeroed: tag 0 never matches (epochs start at 1)
  if ((rc = h->alloc(&p.x, d.d_model / 2)) || (rc = h->alloc(&p.xres, d.d_model)) ||
      (rc = h->alloc(&p.qkv, (size_t)(d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim)) ||
      (rc = h->alloc(&p.attn_out, (size_t)d.n_q_heads * d.head_dim / 2)) || (rc = h->alloc(&p.act, d.ffn / 2)) ||
      (rc = h->alloc(&p.attn_part, (size_t)d.n_kv_heads * pl.kv_chunks_max * G * (d.head_dim + 2))) ||
      (rc = h->alloc(&p.am, 2 * (size_t)grid)) ||
      (rc = h->alloc(&p.ctr, pl.n_counters)) || (rc = h->alloc(&p.attn_ticket, (size_t)L * d.n_kv_heads)) ||
      (rc = h->alloc(&p.am_ticket, 1)) || (rc = h->alloc(&p.abort_flag, 1)))
    return fail(rc);
  if (h->opt.trace) {
    if ((rc = h->alloc(&p.trace, (size_t)grid * h->max_tasks_per_cta * AMK_TRACE_WORDS))) return fail(rc);
  }
  Task* tasks_d;
  int* off_d;
  if ((rc = h->upload(&tasks_d, pl.tasks)) || (rc = h->upload(&off_d, pl.off))) return fail(rc);
  p.tasks = tasks_d;
  p.task_off = off_d;
  for (const StageList& st : pl.stages) {
    DeviceStage ds{st.op, st.layer, nullptr, nullptr};
    if ((rc = h->upload(&ds.tasks, st.tasks)) || (rc = h->upload(&ds.off, st.off))) return fail(rc);
    h->stages.push_back(ds);
  }
  if ((e = cudaHostAlloc(&h->status_host, sizeof(uint32_t), cudaHostAllocMapped)) != cudaSuccess)
    return fail(cuda_fail(e, "cudaHostAlloc"));
  *h->status_host = 0;
  uint32_t* status_dev = nullptr;
  if ((e = cudaHostGetDevicePointer((void**)&status_dev, h->status_host, 0)) != cudaSuccess)
    return fail(cuda_fail(e, "cudaHostGetDevicePointer"));
  p.status = status_dev;
  if ((e = cudaDeviceSynchronize()) != cudaSuccess) return fail(cuda_fail(e, "cudaDeviceSynchronize"));

  *out = h;
  return AMK_OK;
}

void amk_destroy(amk_handle* h) { delete h; }

static int check_step_args(amk_handle* h, int token_id, int pos, int* next_token_out) {
  if (!h || !next_token_out) return AMK_ERR_INVALID_ARG;
  if (pos < 0 || pos >= h->dims.max_seq) return AMK_ERR_INVALID_ARG;
  if (token_id < -1 || token_id >= h->dims.vocab) return AMK_ERR_INVALID_ARG;
  if (*reinterpret_cast<volatile uint32_t*>(h->status_host) != 0) return AMK_ERR_DEVICE_TIMEOUT;
  return AMK_OK;
}

int amk_decode_step(amk_handle* h, int token_id, int pos, float* logits_out, int* next_token_out, void* stream) {
  int rc = check_step_args(h, token_id, pos, next_token_out);
  if (rc) return rc;
  Params p = h->base;
  p.epoch = ++h->epoch;
  p.tag_epoch = p.epoch;
  p.token = token_id;
  p.pos = pos;
  p.logits = logits_out;
  p.next_token = next_token_out;
  p.sync = 1;
  cudaError_t e = launch_decode(p, static_cast<cudaStream_t>(stream), true);
  return e == cudaSuccess ? AMK_OK : cuda_fail(e, "cudaLaunchCooperativeKernel");
}

int amk_decode_step_unfused(amk_handle* h, int token_id, int pos, float* logits_out, int* next_token_out,
                            void* stream) {
  int rc = check_step_args(h, token_id, pos, next_token_out);
  if (rc) return rc;
  Params p = h->base;
  p.epoch = ++h->epoch;   // one tag epoch for all of this step's launches
  p.tag_epoch = p.epoch;
  p.token = token_id;
  p.pos = pos;
  p.logits = logits_out;
  p.next_token = next_token_out;
  p.sync = 0;
  p.trace = nullptr;
  for (const DeviceStage& st : h->stages) {
    p.tasks = st.tasks;
    p.task_off = st.off;
    cudaError_t e = launch_decode(p, static_cast<cudaStream_t>(stream), false);
    if (e != cudaSuccess) return cuda_fail(e, "unfused launch");
  }
  return AMK_OK;
}

int amk_status(const amk_handle* h, uint32_t* detail) {
  if (!h) return AMK_ERR_INVALID_ARG;
  uint32_t s = *reinterpret_cast<volatile uint32_t*>(h->status_host);
  if (detail) *detail = s & 0x7fffffffu;
  return s ? AMK_ERR_DEVICE_TIMEOUT : AMK_OK;
}

int amk_plan_info_get(const amk_handle* h, amk_plan_info* out) {
  if (!h || !out) return AMK_ERR_INVALID_ARG;
  out->grid = h->plan.grid;
  out->threads = kThreads;
  out->smem_bytes = kSmemBytes;
  out->n_tasks = (int)h->plan.tasks.size();
  out->n_counters = h->plan.n_counters;
  out->kv_chunks_max = h->plan.kv_chunks_max;
  out->weight_bytes = amk_step_bytes(&h->dims, 0) - 2ull * h->dims.n_layers * h->dims.n_kv_heads * h->dims.head_dim * 2;
  return AMK_OK;
}

int amk_trace_read(amk_handle* h, uint64_t* out, int max_records) {
  if (!h || !out || max_records < 0) return AMK_ERR_INVALID_ARG;
  if (!h->base.trace) return 0;
  int n = std::min(max_records, h->plan.grid * h->max_tasks_per_cta);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpy(out, h->base.trace, (size_t)n * AMK_TRACE_WORDS * sizeof(uint64_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  return n;
}

}  // extern "C"
