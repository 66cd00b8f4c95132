// Device code of libamk (sm_100a): the persistent decode kernel, its routines, and the weight packer.
//
// One CTA per SM, compute warps + 1: the last warp is the producer, whose elected lane streams every byte this CTA
// will read into a kSlots x kSlotBytes shared-memory ring: weight rows of its GEMV tasks with
// cp.async.bulk, the keys and values of its attention chunk as 128-byte-swizzled tensor boxes with
// cp.async.bulk.tensor; completion is tracked by one mbarrier per slot and at most kInflight copies
// are outstanding at once, while the same lane warms L2 with the items that follow. The producer
// never waits on other CTAs, so the next tasks' weights arrive while the compute warps wait on a
// counter: this is the "prefetch the next layer's weights while the current layer computes" of
// "AutoMegaKernel: A Statically-Checked Agent Harness for Self-Retargeting Megakernel Synthesis"
// (README summary), with dependencies carried by counters instead of grid barriers (technical
// summary, "Methodology", Layer 0: wait -> dispatch -> signal on monotonic counters).
//
// Hand-offs between CTAs carry no memory fence: every vector one CTA passes to others goes out in
// tagged 64-bit words (see tag_of), a reader re-reads any word whose tag is not the one it expects,
// and a stage counter, bumped with a relaxed reduction, only tells readers of a wide vector when to
// start (a gpu-scope release fence would wait on the SM's in-flight weight copies: several
// microseconds per stage under the full stream).
//
// The other warps compute. Every wait is bounded by a %globaltimer deadline; when one expires the CTA
// raises a device abort flag plus a host-visible status word and every later wait returns at once,
// so the launch always completes (outputs are then garbage and the handle reports it).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "amk_internal.h"

namespace amk {
namespace dev {

// ------------------------------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking probe of a phase (try_wait may suspend the thread for a system-defined time).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
// One tile of a 2-D tensor map (x: column, a multiple of 16 bytes; y: row) into shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;"
      ::"r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory"); }
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
__device__ __forceinline__ uint32_t ld_volatile(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void red_relaxed_add(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_relaxed_add(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// Tagged pairs: {fp32 value bits (low word), tag (high word)} as one aligned 64-bit element. Loads
// go to L2 (.cg: never a stale L1 line) on every call.
__device__ __forceinline__ uint64_t pair_of(float v, uint32_t tag) {
  return (uint64_t)__float_as_uint(v) | ((uint64_t)tag << 32);
}
__device__ __forceinline__ void st_pair(uint64_t* p, float v, uint32_t tag) {
  asm volatile("st.global.cg.u64 [%0], %1;" ::"l"(p), "l"(pair_of(v, tag)) : "memory");
}
__device__ __forceinline__ void st_pair2(uint64_t* p, float a, float b, uint32_t tag) {   // 16-byte aligned
  asm volatile("st.global.cg.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(pair_of(a, tag)), "l"(pair_of(b, tag)) : "memory");
}
__device__ __forceinline__ uint2 ld_pair(const uint64_t* p) {   // {value bits, tag}
  uint64_t w;
  asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return make_uint2((uint32_t)w, (uint32_t)(w >> 32));
}
__device__ __forceinline__ uint4 ld_pair2(const uint64_t* p) {   // two pairs, 16-byte aligned: {v0, t0, v1, t1}
  uint64_t a, b;
  asm volatile("ld.global.cg.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
  return make_uint4((uint32_t)a, (uint32_t)(a >> 32), (uint32_t)b, (uint32_t)(b >> 32));
}
__device__ __forceinline__ bool tags_ok(uint4 v, uint32_t tag) { return v.y == tag && v.w == tag; }
// A tagged word of two bf16 values (round to nearest even).
__device__ __forceinline__ uint64_t bf2_word(float a, float b, uint32_t tag);
// Two tagged words (16-byte aligned) through L1: readers use this right after an acquire poll of
// the stage counter (which drops stale L1 lines), so the row partitions of a CTA that read the same
// words share one L2 request.
__device__ __forceinline__ uint4 ld_words2_ca(const uint64_t* p) {
  uint64_t a, b;
  asm volatile("ld.global.ca.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
  return make_uint4((uint32_t)a, (uint32_t)(a >> 32), (uint32_t)b, (uint32_t)(b >> 32));
}
__device__ __forceinline__ uint2 ld_word_ca(const uint64_t* p) {
  uint64_t w;
  asm volatile("ld.global.ca.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return make_uint2((uint32_t)w, (uint32_t)(w >> 32));
}

__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }
__device__ __forceinline__ uint16_t f2bf(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// acc += {lo, hi} * {a0, a1} with one packed fp32 FMA
__device__ __forceinline__ void ffma2(unsigned long long& acc, float lo, float hi, float a0, float a1) {
  asm("{\n\t.reg .b64 wv, av;\n\t"
      "mov.b64 wv, {%1, %2};\n\t"
      "mov.b64 av, {%3, %4};\n\t"
      "fma.rn.f32x2 %0, wv, av, %0;\n\t}"
      : "+l"(acc)
      : "f"(lo), "f"(hi), "f"(a0), "f"(a1));
}
// (o0, o1) += p * (v0, v1) as one packed fp32 FMA.
__device__ __forceinline__ void ffma2_pair(float& o0, float& o1, float p, float v0, float v1) {
  asm("{\n\t.reg .b64 ov, pv, vv;\n\t"
      "mov.b64 ov, {%0, %1};\n\t"
      "mov.b64 pv, {%2, %2};\n\t"
      "mov.b64 vv, {%3, %4};\n\t"
      "fma.rn.f32x2 ov, pv, vv, ov;\n\t"
      "mov.b64 {%0, %1}, ov;\n\t}"
      : "+f"(o0), "+f"(o1)
      : "f"(p), "f"(v0), "f"(v1));
}
__device__ __forceinline__ float f2sum(unsigned long long v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo + hi;
}

// ------------------------------------------------------------------------------------------------
// Shared memory

struct Misc {
  int token;
  int flag;
  float red[kConsumerWarps];
  float am_v[kConsumerWarps];
  int am_i[kConsumerWarps];
  float lm_v;
  int lm_i;
};
static_assert(sizeof(Misc) + 2 * kSlots * 8 <= kMiscBytes, "misc region");
static_assert(sizeof(Task) * kTaskCache == kTaskCacheBytes, "task cache region");

struct Smem {
  uint8_t* ring;
  float* part;
  float* aux;
  float* scale;
  uint64_t* full;
  uint64_t* empty;
  Misc* misc;
};

extern __shared__ __align__(1024) uint8_t smem_raw[];   // 1024: the 128-byte swizzle's period
__device__ __forceinline__ Smem smem_view();

__device__ __forceinline__ Smem carve(uint8_t* base) {
  Smem s;
  s.ring = base;
  s.part = reinterpret_cast<float*>(base + kRingBytes);
  s.aux = reinterpret_cast<float*>(base + kRingBytes + kPartBytes);
  s.scale = reinterpret_cast<float*>(base + kRingBytes + kPartBytes + kAuxBytes);
  uint8_t* m = base + kRingBytes + kPartBytes + kAuxBytes + kScaleBytes;
  s.full = reinterpret_cast<uint64_t*>(m);
  s.empty = s.full + kSlots;
  s.misc = reinterpret_cast<Misc*>(m + 2 * kSlots * 8);
  return s;
}
// The shared-memory view of this CTA, rebuilt from the dynamic shared-memory base (cheap pointer
// arithmetic), so routines take no Smem argument that would otherwise live in local memory.
__device__ __forceinline__ Smem smem_view() { return carve(smem_raw); }

// ------------------------------------------------------------------------------------------------
// Failure handling and waits

__device__ void raise_abort(const Params& p, uint32_t detail) {
  if (atomicCAS(p.abort_flag, 0u, 1u) == 0u) {
    *p.status = 0x80000000u | detail;
    __threadfence_system();
  }
}

// Thread 0 of the compute warps spins until counter >= target (mod 2^32), bounded by the timeout.
// Returns false if the wait expired or another CTA aborted (the caller then carries on: data are
// garbage but every thread keeps the same control flow, so the launch still completes). The count
// only says when the tagged inputs are worth reading; its acquire loads (cheap: it is the writer's
// release that waits on the SM's in-flight copies) also drop this SM's stale L1 lines, so the
// inputs can then be read through L1.
__device__ bool spin_counter(const Params& p, int ctr, uint32_t target) {
  const uint32_t* c = p.ctr + ctr;
  if ((int32_t)(ld_acquire(c) - target) >= 0) return true;
  if (ld_volatile(p.abort_flag)) return false;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(20);
    if ((int32_t)(ld_acquire(c) - target) >= 0) return true;
    if ((it & 15) == 0) {
      if (ld_volatile(p.abort_flag)) return false;
      if (globaltimer() - t0 > p.timeout_ns) {
        raise_abort(p, (1u << 16) | (uint32_t)ctr);
        return false;
      }
    }
  }
}

// All compute threads call this; thread 0 waits, then the compute barrier publishes it.
__device__ __forceinline__ void wait_counter(const Params& p, int ctr, uint32_t mult) {
  if (threadIdx.x == 0) spin_counter(p, ctr, p.epoch * mult);
  bar_compute();
}

// The caller has passed a compute barrier after the task's last tagged store. The count carries no
// data (readers check the tags), so it needs no release: a relaxed reduction.
__device__ __forceinline__ void signal_counter(const Params& p, int ctr) {
  if (threadIdx.x == 0) red_relaxed_add(p.ctr + ctr, 1u);
}

// Re-reads, all together, the 16-byte loads (two tagged pairs each) of `v` whose bit is set in
// `stale` until both tags of each are `tag`: the slow path of a reader that outran the writers'
// stores (no fence orders them before the counter), one round trip per round. Bounded by the
// timeout; after an abort it returns at once with what it read. `addr(j)` is load j's address.
template <int N, class Addr>
__device__ __forceinline__ void repoll2(const Params& p, uint4 (&v)[N], uint32_t stale, uint32_t tag, Addr addr) {
  const uint64_t t0 = globaltimer();
  for (uint32_t round = 1; stale; ++round) {
    __nanosleep(32);
#pragma unroll
    for (int j = 0; j < N; ++j)
      if (stale & (1u << j)) v[j] = ld_pair2(addr(j));
#pragma unroll
    for (int j = 0; j < N; ++j)
      if ((stale & (1u << j)) && tags_ok(v[j], tag)) stale &= ~(1u << j);
    if (stale && (round & 7) == 0) {
      if (ld_volatile(p.abort_flag)) return;
      if (globaltimer() - t0 > p.timeout_ns) {
        raise_abort(p, 6u << 16);
        return;
      }
    }
  }
}
// The same for single 8-byte pairs ({value bits, tag} in x, y).
template <int N, class Addr>
__device__ __forceinline__ void repoll1(const Params& p, uint2 (&v)[N], uint32_t stale, uint32_t tag, Addr addr) {
  const uint64_t t0 = globaltimer();
  for (uint32_t round = 1; stale; ++round) {
    __nanosleep(32);
#pragma unroll
    for (int j = 0; j < N; ++j)
      if (stale & (1u << j)) v[j] = ld_pair(addr(j));
#pragma unroll
    for (int j = 0; j < N; ++j)
      if ((stale & (1u << j)) && v[j].y == tag) stale &= ~(1u << j);
    if (stale && (round & 7) == 0) {
      if (ld_volatile(p.abort_flag)) return;
      if (globaltimer() - t0 > p.timeout_ns) {
        raise_abort(p, 6u << 16);
        return;
      }
    }
  }
}

// Bounded wait on a ring mbarrier phase. Its bound is 4x the counter bound, so a stalled counter is
// always reported first (the ring drains once the counter waits give up); this one only expires if
// the copy protocol itself broke.
__device__ __forceinline__ void wait_slot(const Params& p, uint64_t* bar, uint32_t parity, uint32_t detail) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 4 * p.timeout_ns) {
      raise_abort(p, detail);
      return;
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Byte stream of one task (shared by the producer and the compute warps so both walk the same
// sequence of ring slots).

__device__ __forceinline__ const void* gemv_weights(const Params& p, int op, int l) {
  switch (op) {
    case OP_QKV: return p.layers[l].wqkv;
    case OP_O: return p.layers[l].wo;
    case OP_GU: return p.layers[l].wgu;
    case OP_DOWN: return p.layers[l].wdown;
    default: return p.lm_w;
  }
}
__device__ __forceinline__ const uint16_t* gemv_scales(const Params& p, int op, int l) {
  switch (op) {
    case OP_QKV: return p.layers[l].sqkv;
    case OP_O: return p.layers[l].so;
    case OP_GU: return p.layers[l].sgu;
    case OP_DOWN: return p.layers[l].sdown;
    default: return p.lm_s;
  }
}
__device__ __forceinline__ bool is_gemv(int op) { return op == OP_QKV || op == OP_O || op == OP_GU || op == OP_DOWN || op == OP_LM; }

// ------------------------------------------------------------------------------------------------
// Producer

// Walks the byte stream of one CTA's task list, one ring slot (item) at a time. An item is one
// contiguous weight range (GEMV rows) or a K range plus the matching V range (attention).
struct ItemCursor {
  int ti = 0;       // task index
  int sub = 0;      // GEMV: first row of the item; ATTN: first position of the item
  bool started = false;
  int end = 0;      // GEMV: rows; ATTN: chunk end position
  const uint8_t* base = nullptr;   // GEMV: the task's first weight row, read once per task (the layer's
  int rb = 0, rs = 0;              //   pointer is a dependent global load); row bytes, rows per slot
};

// Item range of a task: GEMV rows [0, t.b), or the positions [begin, end) of an attention chunk
// (empty when the chunk is inactive at this position); other tasks stream nothing.
__device__ __forceinline__ void task_range(const Params& p, const Task& t, int& begin, int& end) {
  begin = end = 0;
  if (t.op == OP_ATTN) {
    const int P = p.pos + 1;
    const int C = attn_num_chunks(P, p.kv_block, attn_chunk_cap(P, p.kv_chunks_max, p.kv_chunks_short));
    if (t.b < C) attn_chunk_range(P, C, t.b, &begin, &end);
  } else if (is_gemv(t.op)) {
    end = t.b;
  }
}

// Advances `c` to the next item; returns false at the end of the list. (src0, n0) and (src1, n1)
// are the item's byte ranges (n1 = 0 for GEMV items; n0 = n1 = 0 for an attention block that holds
// only the current position, which is written this step and patched in shared memory).
__device__ bool next_item(const Params& p, const Task* tasks, int nt, ItemCursor& c, const uint8_t*& src0,
                          uint32_t& n0, const uint8_t*& src1, uint32_t& n1, int& trow, int& tn) {
  while (c.ti < nt) {
    const Task& t = tasks[c.ti];
    if (!c.started) {
      c.started = true;
      task_range(p, t, c.sub, c.end);
      if (is_gemv(t.op) && c.sub < c.end) {
        const GemvGeom& g = p.geom[gemv_slot_of(t.op)];
        c.rb = g.rb;
        c.rs = g.rs;
        c.base = static_cast<const uint8_t*>(gemv_weights(p, t.op, t.layer)) + (size_t)t.a * g.rb;
      }
    }
    if (c.sub < c.end) {
      if (t.op == OP_ATTN) {
        const int nps = attn_positions_per_slot(p.hd);
        const int blk = c.sub, be = min(blk + nps, c.end);
        const int ntma = max(0, min(be, p.pos) - blk);
        const size_t row = ((size_t)t.layer * p.Hkv + t.a) * p.max_seq + blk;
        const size_t off = row * p.hd;
        // the contiguous rows already in the cache (for the L2 warm-up); the copy itself moves
        // 16-row tensor boxes of rows blk..be-1 (the current position's row is patched in later)
        src0 = reinterpret_cast<const uint8_t*>(p.kcache + off);
        src1 = reinterpret_cast<const uint8_t*>(p.vcache + off);
        n0 = n1 = (uint32_t)ntma * (uint32_t)p.hd * 2u;
        trow = (int)row;
        tn = be - blk;
        c.sub = be;
      } else {
        const int n = min(c.rs, c.end - c.sub);
        src0 = c.base + (size_t)c.sub * c.rb;
        n0 = (uint32_t)n * (uint32_t)c.rb;
        src1 = nullptr;
        n1 = 0;
        tn = 0;
        c.sub += n;
      }
      return true;
    }
    ++c.ti;
    c.started = false;
  }
  return false;
}

__device__ __forceinline__ void prefetch_line_l2(const void* a) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(a) : "memory");
}
__device__ __forceinline__ void prefetch_bulk_l2(const void* a, uint32_t bytes) {   // 16-B aligned, 16-B multiple
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(bytes) : "memory");
}


// L2 prefetch of the small static data a task reads on its critical path (row scales, RMSNorm gain,
// this position's RoPE row, the embedding row), issued when the producer starts streaming the
// task's weights, i.e. several ring slots before the compute warps reach it. Under a full HBM
// stream an L2 miss costs microseconds, so these would otherwise stall every stage transition.
__device__ void prefetch_side_data(const Params& p, const Task& t, int token) {
  if (!is_gemv(t.op)) return;
  const uint16_t* sc = gemv_scales(p, t.op, t.layer);
  if (p.wdtype != AMK_W_BF16 && sc && t.b > 0) {
    const char* b = reinterpret_cast<const char*>(sc + t.a);
    const int bytes = t.b * 2;
    for (int o = 0; o < bytes; o += 128) prefetch_line_l2(b + o);
    prefetch_line_l2(b + bytes - 1);
  }
  const uint16_t* gain = t.op == OP_QKV ? p.layers[t.layer].attn_norm
                       : t.op == OP_GU ? p.layers[t.layer].ffn_norm
                       : t.op == OP_LM ? p.final_norm : nullptr;
  if (gain) prefetch_bulk_l2(gain, (uint32_t)p.d * 2);
  if (t.op == OP_QKV) {
    prefetch_bulk_l2(p.rope + (size_t)p.pos * p.hd, (uint32_t)p.hd * 4);
    if (t.layer == 0) prefetch_bulk_l2(p.embed + (size_t)token * p.d, (uint32_t)p.d * 2);
  }
}

// Producer lane: issues every item of the CTA's byte stream into the ring in order, gated only by

// the ring's empty barriers (never by other CTAs).
__device__ __noinline__ void producer(const Params& p, const Task* tasks, int nt) {
  Smem s = smem_view();
  if (smem_u32(s.ring) & 1023u) {   // the swizzled tensor copies need the 1024-byte period
    raise_abort(p, 7u << 16);
    return;
  }
  const uint64_t pol = policy_evict_first();
  int token = p.token;
  if (token < 0) token = __ldcg(p.next_token);
  if (token < 0 || token >= p.V) token = 0;
  ItemCursor cur, pfc;
  uint32_t it = 0, pf_it = 0;
  int last_task = -1;
  const uint8_t *a0, *a1;
  uint32_t n0, n1;
  int trow, tn;
  uint64_t last_pf = 0;
  bool first_item = false;
  while (next_item(p, tasks, nt, cur, a0, n0, a1, n1, trow, tn)) {
    if (cur.ti != last_task) {
      last_task = cur.ti;
      first_item = true;
      prefetch_side_data(p, tasks[cur.ti], token);
    }
    const int slot = it % kSlots;
    if (kPfItems > 0 && pf_it <= it) {   // the L2 warm-up cursor restarts just past this item
      pfc = cur;
      pf_it = it + 1;
    }
    if (it >= (uint32_t)kSlots) {
      const uint32_t par = ((it / kSlots) - 1) & 1;
      if (kPfItems > 0 && !mbar_try_wait(&s.empty[slot], par)) {
        // the slot's previous item has landed but is still held: once that lasts kStallNs the
        // compute warps are waiting on a counter, so warm L2 with what follows, paced
        const uint64_t t0 = globaltimer();
        uint64_t& last = last_pf;
        bool cur_warm = pf_it > it + 1;   // already warmed as a look-ahead item of an earlier stall
        // non-blocking probes: a suspended try_wait would hold the producer past the warm-up times
        while (!mbar_test_wait(&s.empty[slot], par)) {
          __nanosleep(100);
          const uint64_t now = globaltimer();
          if (now - t0 > 4 * p.timeout_ns) {
            raise_abort(p, (3u << 16) | slot);
            break;
          }
          if (now - t0 > kStallNs && now - last > kPfGapNs && pf_it < it + kPfItems &&
              mbar_test_wait(&s.full[slot], par)) {
            const uint8_t *b0, *b1;
            uint32_t m0, m1;
            int r0, rn;
            if (!cur_warm) {   // this item first: it is copied as soon as the slot frees
              if (n0) prefetch_bulk_l2(a0, n0);
              if (n1) prefetch_bulk_l2(a1, n1);
              cur_warm = true;
              last = now;
            } else if (next_item(p, tasks, nt, pfc, b0, m0, b1, m1, r0, rn)) {
              if (m0) prefetch_bulk_l2(b0, m0);
              if (m1) prefetch_bulk_l2(b1, m1);
              ++pf_it;
              last = now;
            } else {
              pf_it = 0xffffffffu;
            }
          }
        }
      } else {
        wait_slot(p, &s.empty[slot], par, (3u << 16) | slot);
      }
    }
    if (kInflight < kSlots && it >= (uint32_t)kInflight) {
      // item it - kInflight must have landed; its slot cannot have been refilled yet (that needs
      // item it - kInflight + kSlots > it), so the parity names that item's phase alone
      const uint32_t j = it - kInflight;
      wait_slot(p, &s.full[j % kSlots], (j / kSlots) & 1, (5u << 16) | (j % kSlots));
    }
    if (first_item && p.trace) {   // the producer's view of the task: its first item is issued now
      p.trace[((size_t)blockIdx.x * p.max_tasks_per_cta + cur.ti) * AMK_TRACE_WORDS + 8] = globaltimer();
      first_item = false;
    }
    if (tn > 0) {
      // attention keys and values: each 64-column half as 64-row boxes, the last rows as 16-row
      // boxes (rows past the item are loaded too and masked by the consumer), 128-byte swizzled
      const int nbig = tn >> 6, nsmall = ((tn & 63) + 15) >> 4, nh = p.hd >> 6;
      const int nps = attn_positions_per_slot(p.hd);
      uint8_t* const kb = s.ring + slot * kSlotBytes;
      mbar_expect_tx(&s.full[slot], (uint32_t)nh * 2u * (uint32_t)(nbig * 8192 + nsmall * 2048));
      for (int hh = 0; hh < nh; ++hh) {
        for (int b = 0; b < nbig + nsmall; ++b) {
          const bool big = b < nbig;
          const int r = big ? 64 * b : 64 * nbig + 16 * (b - nbig);
          const uint32_t o = (uint32_t)(hh * nps * 128 + r * 128);
          tma_load_2d(kb + o, &p.kmap[big ? 0 : 1], hh * 64, trow + r, &s.full[slot], pol);
          tma_load_2d(kb + kSlotBytes / 2 + o, &p.vmap[big ? 0 : 1], hh * 64, trow + r, &s.full[slot], pol);
        }
      }
    } else if (n0 + n1 > 0) {
      mbar_expect_tx(&s.full[slot], n0 + n1);
      bulk_g2s(s.ring + slot * kSlotBytes, a0, n0, &s.full[slot], pol);
      if (n1) bulk_g2s(s.ring + slot * kSlotBytes + kSlotBytes / 2, a1, n1, &s.full[slot], pol);
    } else {
      mbar_arrive(&s.full[slot]);
    }
    if (p.trace && cur.sub >= cur.end)   // the task's last item is issued
      p.trace[((size_t)blockIdx.x * p.max_tasks_per_cta + cur.ti) * AMK_TRACE_WORDS + 9] = globaltimer();
    ++it;
    // the warm-up also runs between stalls, one item per kPfGapNs and at most kPfItems ahead of
    // the ring, so HBM already streams what the ring copies next (they then mostly hit L2)
    if (kPfContinuous && kPfItems > 0 && pf_it < it + kPfItems && pf_it != 0xffffffffu) {
      const uint64_t now = globaltimer();
      if (now - last_pf > kPfGapNs) {
        const uint8_t *b0, *b1;
        uint32_t m0, m1;
        int r0, rn;
        if (pf_it <= it) { pfc = cur; pf_it = it; }
        if (next_item(p, tasks, nt, pfc, b0, m0, b1, m1, r0, rn)) {
          if (m0) prefetch_bulk_l2(b0, m0);
          if (m1) prefetch_bulk_l2(b1, m1);
          ++pf_it;
          last_pf = now;
        } else {
          pf_it = 0xffffffffu;
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// GEMV

// Block-wide sum over the compute threads in a fixed order (deterministic).
// Sum of 4 per-lane values for 4 rows over the warp; lanes with (lane & 7) == 0 return row
// (lane >> 3) & 3's total (transposed butterfly: 6 shuffles for 4 rows).
__device__ __forceinline__ float reduce4_rows(float a0, float a1, float a2, float a3) {
  const int lane = threadIdx.x & 31;
  const bool u16 = lane & 16;
  float k0 = u16 ? a2 : a0, t0 = u16 ? a0 : a2;
  float k1 = u16 ? a3 : a1, t1 = u16 ? a1 : a3;
  k0 += __shfl_xor_sync(0xffffffffu, t0, 16);
  k1 += __shfl_xor_sync(0xffffffffu, t1, 16);
  const bool u8 = lane & 8;
  float u = u8 ? k1 : k0, v = u8 ? k0 : k1;
  u += __shfl_xor_sync(0xffffffffu, v, 8);
  u += __shfl_xor_sync(0xffffffffu, u, 4);
  u += __shfl_xor_sync(0xffffffffu, u, 2);
  u += __shfl_xor_sync(0xffffffffu, u, 1);
  return u;
}

// Sum of 2 per-lane values for 2 rows over the warp; lanes 0..15 return row 0's total and lanes
// 16..31 row 1's (transposed butterfly: 5 shuffles for 2 rows).
__device__ __forceinline__ float reduce2_rows(float a0, float a1) {
  const int lane = threadIdx.x & 31;
  const bool u16 = lane & 16;
  float k = u16 ? a1 : a0;
  k += __shfl_xor_sync(0xffffffffu, u16 ? a0 : a1, 16);
  k += __shfl_xor_sync(0xffffffffu, k, 8);
  k += __shfl_xor_sync(0xffffffffu, k, 4);
  k += __shfl_xor_sync(0xffffffffu, k, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

template <int GB>
struct GroupWords { static constexpr int N = GB >= 4 ? GB / 4 : 1; };

// One thread's group of GB weight bytes of a row: 16-byte vector loads (GB >= 16) or one smaller one.
template <int GB>
__device__ __forceinline__ void lds_group(const uint8_t* ptr, uint32_t (&w)[GroupWords<GB>::N]) {
  if constexpr (GB >= 16) {
#pragma unroll
    for (int i = 0; i < GB / 16; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(ptr)[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (GB == 8) {
    const uint2 v = *reinterpret_cast<const uint2*>(ptr);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (GB == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(ptr);
  } else {
    w[0] = *reinterpret_cast<const uint16_t*>(ptr);
  }
}

// int8 chunk of ECH elements against int16 activations: exact int32 dot product with dp2a (two
// int16 x int8 products per instruction; .lo takes weight bytes 0-1, .hi bytes 2-3). Activation word k
// holds elements 2k (low half) and 2k+1 (high half).
template <int ECH>
__device__ __forceinline__ int dot_chunk_i8(int acc, const uint32_t* w, const uint32_t* a) {
  if constexpr (ECH >= 4) {
#pragma unroll
    for (int k = 0; k < ECH / 4; ++k) {
      acc = __dp2a_lo((int)a[2 * k], (int)w[k], acc);
      acc = __dp2a_hi((int)a[2 * k + 1], (int)w[k], acc);
    }
  } else {
    acc = __dp2a_lo((int)a[0], (int)w[0], acc);
  }
  return acc;
}

// dp2a of two signed 16-bit halves of a with two unsigned bytes of b (low or high byte pair).
__device__ __forceinline__ int dp2a_lo_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Vector loads of N consecutive fp32 elements (N in {2, 4, 8, 16}) through L1.
template <int N>
__device__ __forceinline__ void ld_f32_ca(const float* p, float* o) {
  if constexpr (N >= 4) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const float4 v = __ldca(reinterpret_cast<const float4*>(p) + i);
      o[4 * i] = v.x; o[4 * i + 1] = v.y; o[4 * i + 2] = v.z; o[4 * i + 3] = v.w;
    }
  } else {
    const float2 v = __ldca(reinterpret_cast<const float2*>(p));
    o[0] = v.x; o[1] = v.y;
  }
}
template <int N>
__device__ __forceinline__ void ld_bf16_words(const uint16_t* p, uint32_t* o) {   // read-only: N/2 words
  if constexpr (N >= 8) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      o[4 * i] = v.x; o[4 * i + 1] = v.y; o[4 * i + 2] = v.z; o[4 * i + 3] = v.w;
    }
  } else if constexpr (N == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    o[0] = v.x; o[1] = v.y;
  } else {
    o[0] = __ldg(reinterpret_cast<const unsigned int*>(p));
  }
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ uint64_t bf2_word(float a, float b, uint32_t tag) {
  return (uint64_t)((uint32_t)f2bf(a) | ((uint32_t)f2bf(b) << 16)) | ((uint64_t)tag << 32);
}
__device__ __forceinline__ void st_word(uint64_t* p, uint64_t w) {
  asm volatile("st.global.cg.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Byte offset, inside a row, of piece c of the group that (warp column col, lane) owns. A group of
// GB bytes is min(GB, 16)-byte pieces laid 32 pieces apart, so one load instruction of a warp reads
// 32 x 16 contiguous bytes (no shared-memory bank conflicts).
template <int GB>
__device__ __forceinline__ int piece_offset(int col, int lane, int c) {
  constexpr int PB = GB < 16 ? GB : 16;
  return col * 32 * GB + c * 32 * PB + lane * PB;
}

// One GEMV task: rows [t.a, t.a + t.b) of the op's packed matrix against this step's input vector.
// WK (weight kind): 1 int8 and 2 int4 weights, dp2a against int16 activations quantised per
// 16-byte piece; 0 bf16 weights with packed fp32 FMAs. GB: weight bytes per thread per row; NR:
// compile-time bound on groups per thread (geometry nr <= NR). For RMSNorm inputs the thread works on x * g and the
// 1/rms factor is applied per row in the epilogue, so the input loads need one L2 round trip.
// The hot GEMV instance (int8, 32-byte groups, one group per thread) is inlined into the kernel's
// task loop: a non-inlined call saves and restores registers through local memory, whose lines
// rarely stay in L1 next to 226 KB of shared memory, at every task boundary.
template <int WK>
__device__ __forceinline__ int elem_of_byte(int b) { return WK == 0 ? b / 2 : WK == 1 ? b : b * 2; }

template <int WK, int GB, int NR, bool PART = (WK == 2)>
__device__ __forceinline__ uint32_t gemv_body(const Params& p, const Task t, uint32_t it, int token,
                                             unsigned long long* tr) {
  const Smem s = smem_view();
  constexpr bool IQ = WK != 0;                          // quantised weights: row scales, dp2a
  constexpr int PB = GB < 16 ? GB : 16;                 // bytes per piece
  constexpr int NP = GB / PB;                           // pieces per group
  constexpr int PE = WK == 0 ? PB / 2 : WK == 1 ? PB : PB * 2;   // elements per piece
  constexpr int NB = GB >= 64 ? AMK_NB64 : GB >= 32 ? AMK_NB32 : 4;   // rows per register batch
  constexpr int WPP = PB >= 4 ? PB / 4 : 1;             // weight words per piece
  // The geometry is copied to registers once: it is reached through a generic pointer, and each
  // shared-memory store in the row loop would otherwise force the compiler to read it again.
  const GemvGeom g = p.geom[gemv_slot_of(t.op)];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int op = t.op, l = t.layer, row0 = t.a, nrows = t.b;
  const bool first = t.flags & kFirstOfStage;
  const int rp = warp / g.wpg, wg = warp % g.wpg;
  const bool active = rp < g.rp;
  const bool norm = op == OP_QKV || op == OP_GU || op == OP_LM;

  // ---- static data first, so its latency hides behind the wait: row scales into shared memory,
  //      this thread's RMSNorm gains into registers, this position's RoPE row into aux ----
  const uint16_t* sc = IQ ? gemv_scales(p, op, l) : nullptr;
  if (IQ && sc)
    for (int i = tid; i < nrows; i += kConsumerThreads) s.scale[i] = bf2f(__ldg(sc + row0 + i));
  // pv: this thread's pieces that lie in the row. PART: the last warp of a row may be partly
  // filled, so each piece is checked against the row's end; otherwise whole groups are. Only int4
  // rows can end inside a warp: rows are multiples of 64 elements, so an int8 or bf16 row is a
  // whole number of warps of the smallest group, and the planner picks no larger group that leaves
  // lanes idle when a smaller one fills them.
  bool pv[NR * NP];
  int col[NR];
#pragma unroll
  for (int j = 0; j < NR; ++j) {
    col[j] = j * g.wpg + wg;
    const bool ok = active && j < g.nr && col[j] < g.wg_total;
#pragma unroll
    for (int c = 0; c < NP; ++c) pv[j * NP + c] = PART ? ok && piece_offset<GB>(col[j], lane, c) < g.rb : ok;
  }
  const uint16_t* gain =
      op == OP_QKV ? p.layers[l].attn_norm : op == OP_GU ? p.layers[l].ffn_norm : op == OP_LM ? p.final_norm : nullptr;
  float* const resid_rows = s.aux;   // residual rows (O, down) or the RoPE row (QKV)
  if (op == OP_QKV)
    for (int i = tid; i < p.hd; i += kConsumerThreads) resid_rows[i] = __ldg(p.rope + (size_t)p.pos * p.hd + i);

  // the RMSNorm gain vector (static) into the GEMV partial-sum region before the wait, so the
  // thread's gains come from shared memory after it (no second round trip behind the inputs)
  const int K = g.K;
  const bool gain_smem = norm && K * 2 <= kPartBytes;
  uint16_t* const gsm = reinterpret_cast<uint16_t*>(s.part);
  if (gain_smem)
    for (int i = tid * 8; i < K; i += 8 * kConsumerThreads)
      *reinterpret_cast<uint4*>(gsm + i) = __ldg(reinterpret_cast<const uint4*>(gain + i));

  if (p.sync && first && t.wait_ctr >= 0) wait_counter(p, t.wait_ctr, t.wait_mult);
  else if (gain_smem) bar_compute();
  if (tr && tid == 0) tr[2] = globaltimer();

  // ---- inputs: this thread's own elements (tagged bf16 pairs, read through L1 right after the
  //      acquire poll; any stale word re-read) with their RMSNorm gains and, for O / down, the
  //      residual of the task's rows (fp32 rows this CTA wrote itself), all in one batch of loads ----
  // Row partition 0 covers every input element exactly once, so its threads' squares sum to the
  // RMSNorm statistic; each warp leaves its share in misc->red and the epilogue (behind its own
  // barrier) finishes the sum, so the prologue has a single dependent L2 round trip and no barrier.
  static_assert(kMaxTaskRows <= 2 * kConsumerThreads, "two residual rows per thread");
  const bool resid = op == OP_O || op == OP_DOWN;
  const bool from_embed = op == OP_QKV && l == 0;
  const uint32_t ep = p.tag_epoch;
  // who wrote what: QKV(l) reads x after down(l - 1), GU(l) x after O(l), O(l) the merged attention,
  // DOWN(l) the SwiGLU output, the LM head x after the last down
  const uint64_t* src = op == OP_O ? p.attn_out : op == OP_DOWN ? p.act : p.x;
  const uint32_t tag_in = op == OP_QKV ? tag_of(ep, l - 1, 1) : op == OP_LM ? tag_of(ep, p.L - 1, 1) : tag_of(ep, l, 0);
  // the residual of O(l) is x after down(l - 1) (the embedding row for layer 0), of DOWN(l) x after O(l)
  const uint16_t* erow = p.embed + (size_t)token * p.d;
  float rv0 = 0.f, rv1 = 0.f;
  if (resid) {
    const bool re = op == OP_O && l == 0;
    if (tid < nrows) rv0 = re ? bf2f(__ldg(erow + row0 + tid)) : __ldca(p.xres + row0 + tid);
    if (tid + kConsumerThreads < nrows)
      rv1 = re ? bf2f(__ldg(erow + row0 + tid + kConsumerThreads)) : __ldca(p.xres + row0 + tid + kConsumerThreads);
  }
  // this thread's words: PE / 2 per piece (two bf16 elements each), loaded two at a time
  constexpr int NW = NR * NP * PE / 2;          // words of the thread
  constexpr int NL = PE >= 4 ? NW / 2 : NW;     // 16-byte loads of two words (8-byte loads of one when a piece is 2 elements)
  uint4 wv[NL];
  auto waddr = [&](int k) {   // address of load k: piece k / (loads per piece), its (k % ...)-th pair of words
    constexpr int LPP = PE >= 4 ? PE / 4 : 1;
    const int j = (k / LPP) / NP, c = (k / LPP) % NP;
    return src + elem_of_byte<WK>(piece_offset<GB>(col[j], lane, c)) / 2 + 2 * (k % LPP);
  };
  float ss = 0.f;
  float xv[NR * NP * PE];
  if (from_embed) {
#pragma unroll
    for (int j = 0; j < NR; ++j) {
#pragma unroll
      for (int c = 0; c < NP; ++c) {
        float* xp = &xv[(j * NP + c) * PE];
        const int e = elem_of_byte<WK>(piece_offset<GB>(col[j], lane, c));
        if (pv[j * NP + c]) {
          uint32_t ew[PE / 2];
          ld_bf16_words<PE>(erow + e, ew);
#pragma unroll
          for (int k = 0; k < PE / 2; ++k) { xp[2 * k] = bf_lo(ew[k]); xp[2 * k + 1] = bf_hi(ew[k]); }
        } else {
#pragma unroll
          for (int k = 0; k < PE; ++k) xp[k] = 0.f;
        }
      }
    }
  } else {
    constexpr int LPP = PE >= 4 ? PE / 4 : 1;
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      wv[k] = make_uint4(0u, tag_in, 0u, tag_in);
      if (pv[k / LPP]) {
        if constexpr (PE >= 4) {
          wv[k] = ld_words2_ca(waddr(k));
        } else {
          const uint2 w = ld_word_ca(waddr(k));
          wv[k] = make_uint4(w.x, w.y, 0u, tag_in);
        }
      }
    }
    uint32_t stale = 0;
#pragma unroll
    for (int k = 0; k < NL; ++k)
      if (!tags_ok(wv[k], tag_in)) stale |= 1u << k;
    if (stale) {   // rare: a writer's store had not reached L2; re-read those words from L2
      const uint64_t t0 = globaltimer();
      for (uint32_t round = 1; stale; ++round) {
        __nanosleep(32);
#pragma unroll
        for (int k = 0; k < NL; ++k)
          if (stale & (1u << k)) {
            if constexpr (PE >= 4) {
              wv[k] = ld_pair2(waddr(k));
            } else {
              const uint2 w = ld_pair(waddr(k));
              wv[k] = make_uint4(w.x, w.y, 0u, tag_in);
            }
            if (tags_ok(wv[k], tag_in)) stale &= ~(1u << k);
          }
        if (stale && (round & 7) == 0) {
          if (ld_volatile(p.abort_flag)) break;
          if (globaltimer() - t0 > p.timeout_ns) { raise_abort(p, 6u << 16); break; }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NL; ++k) {   // load k covers elements 4k..4k+3 of the thread (2k, 2k+1 for 2-element pieces)
      if constexpr (PE >= 4) {
        xv[4 * k] = bf_lo(wv[k].x); xv[4 * k + 1] = bf_hi(wv[k].x);
        xv[4 * k + 2] = bf_lo(wv[k].z); xv[4 * k + 3] = bf_hi(wv[k].z);
      } else {
        xv[2 * k] = bf_lo(wv[k].x); xv[2 * k + 1] = bf_hi(wv[k].x);
      }
    }
  }
  if (tr && tid == 0) {   // this thread's inputs landed
    asm volatile("" ::"f"(xv[0]));
    tr[12] = globaltimer();
  }
  if (norm) {
#pragma unroll
    for (int j = 0; j < NR; ++j) {
#pragma unroll
      for (int c = 0; c < NP; ++c) {
        float* xp = &xv[(j * NP + c) * PE];
        if (pv[j * NP + c]) {   // the gains: from shared memory when staged, else a second round trip
          uint32_t gp[PE / 2];
          const int e = elem_of_byte<WK>(piece_offset<GB>(col[j], lane, c));
          if (gain_smem) {
            if constexpr (PE >= 8) {
#pragma unroll
              for (int k = 0; k < PE / 8; ++k) {
                const uint4 w = reinterpret_cast<const uint4*>(gsm + e)[k];
                gp[4 * k] = w.x; gp[4 * k + 1] = w.y; gp[4 * k + 2] = w.z; gp[4 * k + 3] = w.w;
              }
            } else {
#pragma unroll
              for (int k = 0; k < PE / 2; ++k) gp[k] = reinterpret_cast<const uint32_t*>(gsm + e)[k];
            }
          } else {
            ld_bf16_words<PE>(gain + e, gp);
          }
#pragma unroll
          for (int k = 0; k < PE; ++k) ss = fmaf(xp[k], xp[k], ss);
#pragma unroll
          for (int k = 0; k < PE / 2; ++k) { xp[2 * k] *= bf_lo(gp[k]); xp[2 * k + 1] *= bf_hi(gp[k]); }
        }
      }
    }
    if (rp != 0) ss = 0.f;
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s.misc->red[warp] = ss;
  }

  uint32_t ah[IQ ? NR * NP * PE / 2 : 1];
  float asc[IQ ? NR * NP : 1];   // per-piece scale: activation = int16 * asc
  int sa[WK == 2 ? NR * NP : 1];  // int4: per-piece sum of the int16 activations (nibble offset 8)
  if constexpr (IQ) {
#pragma unroll
    for (int c = 0; c < NR * NP; ++c) {
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < PE; ++k) amax = fmaxf(amax, fabsf(xv[c * PE + k]));
      const float q = amax > 0.f ? 32767.f / amax : 0.f;
      asc[c] = amax * (1.f / 32767.f);
      // round(x * q) (|x * q| <= 32767, ties to even) without the quarter-rate float-to-int
      // conversion: the product is rounded to fp32 first (as a conversion of it would be), then
      // adding 1.5 * 2^23 leaves the integer in the low bits of the sum, whose bit pattern is
      // 0x4B400000 + round(x * q); its low 16 bits are the int16 in two's complement
      constexpr float kMagic = 12582912.f;
      constexpr uint32_t kMagicBits = 0x4B400000u;
      auto qb = [&](int k) { return __float_as_uint(__fadd_rn(__fmul_rn(xv[c * PE + k], q), kMagic)); };
      auto pack2 = [](uint32_t lo, uint32_t hi) { return __byte_perm(lo, hi, 0x5410); };   // low halves
      if constexpr (WK == 1) {
#pragma unroll
        for (int k = 0; k < PE / 2; ++k) ah[c * PE / 2 + k] = pack2(qb(2 * k), qb(2 * k + 1));
      } else {
        // a weight word holds elements 8m..8m+7 as nibbles: its low nibbles (elements 0, 2, 4, 6)
        // and high nibbles (1, 3, 5, 7) meet activation words (x0, x2), (x4, x6), (x1, x3), (x5, x7)
        uint32_t bsum = 0u;   // sum of the bit patterns: PE * kMagicBits + the sum of the integers
#pragma unroll
        for (int m = 0; m < PE / 8; ++m) {
          const uint32_t x0 = qb(8 * m), x1 = qb(8 * m + 1), x2 = qb(8 * m + 2), x3 = qb(8 * m + 3);
          const uint32_t x4 = qb(8 * m + 4), x5 = qb(8 * m + 5), x6 = qb(8 * m + 6), x7 = qb(8 * m + 7);
          ah[c * PE / 2 + 4 * m + 0] = pack2(x0, x2);
          ah[c * PE / 2 + 4 * m + 1] = pack2(x4, x6);
          ah[c * PE / 2 + 4 * m + 2] = pack2(x1, x3);
          ah[c * PE / 2 + 4 * m + 3] = pack2(x5, x7);
          bsum += x0 + x1 + x2 + x3 + x4 + x5 + x6 + x7;
        }
        sa[c] = (int)(bsum - (uint32_t)PE * kMagicBits);
      }
    }
  }

  if (resid) {   // read back by other threads in the epilogue, behind its barrier
    if (tid < nrows) resid_rows[tid] = rv0;
    if (tid + kConsumerThreads < nrows) resid_rows[tid + kConsumerThreads] = rv1;
  }
  if (gain_smem) bar_compute();   // every thread has its gains before the rows' partial sums reuse the region
  if (tr && tid == 0) {   // stamped once the (quantised) inputs exist
    if constexpr (IQ) asm volatile("" ::"f"(asc[0]));
    tr[4] = globaltimer();
  }

  // ---- rows, one ring slot at a time ----
  const int blk_rows = g.rs * (kRowBlock / g.rs);
  const int rpg = (g.rs + g.rp - 1) / g.rp;
  float lm_v = -CUDART_INF_F;
  int lm_i = 0x7fffffff;
  int blk_base = 0;                         // task-relative first row of the current epilogue block
  for (int r0 = 0; r0 < nrows; r0 += g.rs, ++it) {
    const int slot = it % kSlots;
    wait_slot(p, &s.full[slot], (it / kSlots) & 1, (2u << 16) | slot);
    if (tr && r0 == 0 && tid == 0) tr[5] = globaltimer();
    const int srows = min(g.rs, nrows - r0);
    const uint8_t* sbuf = s.ring + slot * kSlotBytes;
    if (active) {
      const int rb0 = rp * rpg, re = min(rb0 + rpg, srows);
      for (int r = rb0; r < re; r += NB) {
        float a[NB];
#pragma unroll
        for (int rr = 0; rr < NB; ++rr) {
          float v = 0.f;
          if (r + rr < re) {
            const uint8_t* rowp = sbuf + (size_t)(r + rr) * g.rb;
#pragma unroll
            for (int j = 0; j < NR; ++j) {
              if (pv[j * NP]) {   // a group's pieces are contiguous: the first lies in the row if any does
#pragma unroll
              for (int c = 0; c < NP; ++c) {
                if (!PART || c == 0 || pv[j * NP + c]) {
                  uint32_t w[WPP];
                  lds_group<PB>(rowp + piece_offset<GB>(col[j], lane, c), w);
                  if constexpr (WK == 1) {
                    const int acc = dot_chunk_i8<PE>(0, w, &ah[(j * NP + c) * PE / 2]);
                    v = fmaf((float)acc, asc[j * NP + c], v);
                  } else if constexpr (WK == 2) {
                    // nibbles stored as q + 8: dot(a, u) - 8 * sum(a) = dot(a, q), exact in int32
                    const uint32_t* a4 = &ah[(j * NP + c) * PE / 2];
                    int acc = 0;
#if AMK_I4_NOSHIFT
                    // high nibbles stay in place (16 u, u < 16, as unsigned bytes) in their own sum
                    int acc16 = 0;
#pragma unroll
                    for (int k = 0; k < WPP; ++k) {
                      const uint32_t lo = w[k] & 0x0f0f0f0fu, hi = w[k] & 0xf0f0f0f0u;
                      acc = __dp2a_lo((int)a4[4 * k + 0], (int)lo, acc);
                      acc = __dp2a_hi((int)a4[4 * k + 1], (int)lo, acc);
                      acc16 = dp2a_lo_su(a4[4 * k + 2], hi, acc16);
                      acc16 = dp2a_hi_su(a4[4 * k + 3], hi, acc16);
                    }
                    acc += acc16 >> 4;   // a multiple of 16: the shift is exact
#else
#pragma unroll
                    for (int k = 0; k < WPP; ++k) {
                      const uint32_t lo = w[k] & 0x0f0f0f0fu, hi = (w[k] >> 4) & 0x0f0f0f0fu;
                      acc = __dp2a_lo((int)a4[4 * k + 0], (int)lo, acc);
                      acc = __dp2a_hi((int)a4[4 * k + 1], (int)lo, acc);
                      acc = __dp2a_lo((int)a4[4 * k + 2], (int)hi, acc);
                      acc = __dp2a_hi((int)a4[4 * k + 3], (int)hi, acc);
                    }
#endif
                    acc -= 8 * sa[j * NP + c];
                    v = fmaf((float)acc, asc[j * NP + c], v);
                  } else {
                    unsigned long long acc2 = 0ull;
#pragma unroll
                    for (int k = 0; k < WPP; ++k)
                      ffma2(acc2, bf_lo(w[k]), bf_hi(w[k]), xv[(j * NP + c) * PE + 2 * k], xv[(j * NP + c) * PE + 2 * k + 1]);
                    v += f2sum(acc2);
                  }
                }
              }
              }
            }
          }
          a[rr] = v;
        }
        if constexpr (NB == 1) {
          float tot = a[0];
#pragma unroll
          for (int o = 16; o; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
          if (lane == 0) s.part[wg * kRowBlock + (r0 + r - blk_base)] = tot;
        } else if constexpr (NB == 2) {
          const float tot = reduce2_rows(a[0], a[1]);
          const int row = r + (lane >> 4);
          if ((lane & 15) == 0 && row < re) s.part[wg * kRowBlock + (r0 + row - blk_base)] = tot;
        } else {
          const float tot = reduce4_rows(a[0], a[1], a[2], a[3]);
          const int row = r + ((lane >> 3) & 3);
          if ((lane & 7) == 0 && row < re) s.part[wg * kRowBlock + (r0 + row - blk_base)] = tot;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[slot]);

    // ---- epilogue of a finished block of rows: results go out as tagged pairs ----
    const int done = r0 + srows;
    if (done - blk_base == blk_rows || done == nrows) {
      if (tr && done == nrows && tid == 0) tr[6] = globaltimer();
      bar_compute();
      if (tr && done == nrows && tid == 0) tr[10] = globaltimer();
      float inv = 1.f;
      if (norm) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) t += s.misc->red[w];
        inv = rsqrtf(t / (float)p.d + p.eps);
      }
      const int bs = blk_base, bn = done - blk_base;
      const uint32_t tag_out = tag_of(ep, l, op == OP_DOWN ? 1 : 0);
      auto rowsum = [&](int rr) {
        float acc = 0.f;
        for (int w = 0; w < g.wpg; ++w) acc += s.part[w * kRowBlock + rr];
        acc *= inv;
        return IQ && sc ? acc * s.scale[bs + rr] : acc;
      };
      if (op == OP_GU) {
        // four packed rows (gate, up, gate, up) give two SwiGLU outputs: one bf16 pair
        for (int qd = tid; qd < bn / 4; qd += kConsumerThreads) {
          const float g0 = rowsum(4 * qd), u0 = rowsum(4 * qd + 1), g1 = rowsum(4 * qd + 2), u1 = rowsum(4 * qd + 3);
          const float a0 = g0 / (1.f + __expf(-g0)) * u0, a1 = g1 / (1.f + __expf(-g1)) * u1;
          st_word(p.act + (row0 + bs) / 4 + qd, bf2_word(a0, a1, tag_out));
        }
      } else if (op == OP_QKV) {
        for (int pr = tid; pr < bn / 2; pr += kConsumerThreads) {
          const float v0 = rowsum(2 * pr), v1 = rowsum(2 * pr + 1);
          const int gr = row0 + bs + 2 * pr;
          {
            // packed rows 2i, 2i + 1 of a head are elements i and i + hd/2 of q, k or v: roped q, roped
            // k and v go out in packed order, k and v rounded to bf16 as they are cached at pos
            const int hd = p.hd, head = gr / hd, i = (gr % hd) >> 1;
            float w0 = v0, w1 = v1;
            if (head < p.Hq + p.Hkv) {
              const float c = resid_rows[2 * i], sn = resid_rows[2 * i + 1];
              w0 = v0 * c - v1 * sn;
              w1 = v1 * c + v0 * sn;
            }
            if (head >= p.Hq) {
              const bool is_k = head < p.Hq + p.Hkv;
              uint16_t* kv = (is_k ? p.kcache : p.vcache) +
                             (((size_t)l * p.Hkv + (head - p.Hq - (is_k ? 0 : p.Hkv))) * p.max_seq + p.pos) * hd;
              const uint16_t b0 = f2bf(w0), b1 = f2bf(w1);
              kv[i] = b0;
              kv[i + hd / 2] = b1;
              w0 = bf2f(b0);
              w1 = bf2f(b1);
            }
            st_pair2(p.qkv + gr, w0, w1, tag_out);   // gr even: 16-byte aligned
          }
        }
      } else if (op == OP_LM) {
        for (int rr = tid; rr < bn; rr += kConsumerThreads) {
          const float val = rowsum(rr);
          const int gr = row0 + bs + rr;
          if (p.logits) p.logits[gr] = val;
          if (val > lm_v || (val == lm_v && gr < lm_i)) { lm_v = val; lm_i = gr; }
        }
      } else {
        // O / down: two rows per thread; the fp32 rows stay this CTA's residual, a bf16 pair goes out
        for (int pr = tid; pr < bn / 2; pr += kConsumerThreads) {
          const int gr = row0 + bs + 2 * pr;
          const float x0 = resid_rows[bs + 2 * pr] + rowsum(2 * pr);
          const float x1 = resid_rows[bs + 2 * pr + 1] + rowsum(2 * pr + 1);
          *reinterpret_cast<float2*>(p.xres + gr) = make_float2(x0, x1);
          st_word(p.x + gr / 2, bf2_word(x0, x1, tag_out));
        }
      }
      bar_compute();
      if (tr && done == nrows && tid == 0) tr[11] = globaltimer();
      blk_base = done;
    }
  }

  if (op == OP_LM) {
    // CTA argmax of this task, folded into the CTA's running best
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, lm_v, o);
      const int oi = __shfl_xor_sync(0xffffffffu, lm_i, o);
      if (ov > lm_v || (ov == lm_v && oi < lm_i)) { lm_v = ov; lm_i = oi; }
    }
    if (lane == 0) { s.misc->am_v[warp] = lm_v; s.misc->am_i[warp] = lm_i; }
    bar_compute();
    if (tid == 0) {
      float bv = s.misc->lm_v;
      int bi = s.misc->lm_i;
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float ov = s.misc->am_v[w];
        const int oi = s.misc->am_i[w];
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      s.misc->lm_v = bv;
      s.misc->lm_i = bi;
    }
    bar_compute();
  }
  return it;
}

template <int WK, int GB, int NR>
__device__ __noinline__ uint32_t gemv_task(const Params& p, const Task t, uint32_t it, int token,
                                          unsigned long long* tr) {
  return gemv_body<WK, GB, NR>(p, t, it, token, tr);
}

// Picks the register footprint: one group per thread, or the most the bytes per thread allow
// (<= 32 int8 / 32 bf16 activations per thread).
template <int WK, int GB>
__device__ __forceinline__ uint32_t gemv_nr(const Params& p, const Task& t, uint32_t it, int token,
                                            unsigned long long* tr, int nr) {
  constexpr int NRMAX = (WK == 0 ? 64 : WK == 1 ? 32 : AMK_I4_MAX_GB) / GB;
  if constexpr (NRMAX <= 1) {
    return gemv_task<WK, GB, 1>(p, t, it, token, tr);
  } else {
    if (nr <= 1) return gemv_task<WK, GB, 1>(p, t, it, token, tr);
    return gemv_task<WK, GB, NRMAX>(p, t, it, token, tr);
  }
}

// ------------------------------------------------------------------------------------------------
// Attention (split-KV flash decoding)

// 2^x with the hardware approximation (relative error ~2^-22; 2^-inf = 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float exp2_scale(float m, float M) { return m == -CUDART_INF_F ? 0.f : fast_exp2(m - M); }

// ---- warp-level tensor-core helpers (attention) ----
// D += A B for one m16n8k16 tile: bf16 A (4 registers: rows g / g + 8, k 2t.. / 2t + 8..) and B
// (2 registers: k 2t.. / 2t + 8.., column g), fp32 D (rows g / g + 8, columns 2t, 2t + 1), where g =
// lane / 4 and t = lane % 4.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Four 8x8 bf16 tiles from shared memory; lanes 8i..8i+7 give the row addresses of tile i.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
// Two 8x8 bf16 tiles, transposed; lanes 0..15 give the row addresses.
__device__ __forceinline__ void ldsm_x2_trans(uint32_t& r0, uint32_t& r1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}
// (a, b) as a bf16 pair (a in the low half) plus the bf16 pair of what rounding left over, so that
// hi + lo carries about 16 significant bits of each value.
__device__ __forceinline__ void split_bf2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
  const __nv_bfloat162 l2 = __floats2bfloat162_rn(a - __low2float(h2), b - __high2float(h2));
  hi = *reinterpret_cast<const uint32_t*>(&h2);
  lo = *reinterpret_cast<const uint32_t*>(&l2);
}
// Float <-> int keys whose signed order is the float order (for an integer atomicMax).
__device__ __forceinline__ int max_key(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float key_max(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }
// Byte offset of 16-byte chunk ch (8 elements) of row r of a key or value plane in a ring slot. The
// tensor copies land 64-column halves (128-byte rows, nps rows each) one after the other, with the
// 128-byte swizzle: chunk c of row r sits at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t kv_off(int r, int ch, int nps) {
  return (uint32_t)((ch >> 3) * nps * 128 + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

// Log-sum-exp merge of the C chunk partials (unnormalised o, running max m in log2 units, sum l) of
// KV head h of layer l into the tagged attention output. One thread per (query head, element); a
// warp holds 32 elements of one query head. Per block of 16 chunks, lane k < 16 loads chunk k's
// (m, l) pair of pairs while every lane loads its own element of the 16 chunks' o, all in one batch
// (one L2 round trip: a query head's chunks are hd + 2 pairs apart, so one base address and
// immediate offsets serve every load; stale tags are re-read together); the block max and the
// weighted sum of l are warp reductions and each chunk's weight reaches the other lanes by shuffle.
// Blocks fold into running (M, L, acc) with the usual rescaling, so any C works.
template <int HD>
__device__ __noinline__ void merge_head(const Params& p, int h, int C, int l) {
  constexpr int stride = HD + 2, kBlk = 16;
  const int G = p.Hq / p.Hkv, lane = threadIdx.x & 31;
  const uint32_t tg = tag_of(p.tag_epoch, l);
  for (int idx = threadIdx.x; idx < G * HD; idx += kConsumerThreads) {   // G * HD: whole warps
    const int g = idx / HD, e = idx % HD;
    const uint64_t* pg = p.attn_part + ((size_t)h * G + g) * p.kv_chunks_max * stride;
    float M = -CUDART_INF_F, L = 0.f, acc = 0.f;
    for (int c0 = 0; c0 < C; c0 += kBlk) {
      const int nb = min(kBlk, C - c0);
      const uint64_t* pc = pg + (size_t)c0 * stride;
      uint4 ml[1] = {make_uint4(__float_as_uint(-CUDART_INF_F), tg, 0u, tg)};
      if (lane < nb) ml[0] = ld_pair2(pc + lane * stride + HD);
      uint2 ov[kBlk];
#pragma unroll
      for (int k = 0; k < kBlk; ++k) ov[k] = k < nb ? ld_pair(pc + k * stride + e) : make_uint2(0u, tg);
      if (!tags_ok(ml[0], tg)) repoll2(p, ml, 1u, tg, [&](int) { return pc + lane * stride + HD; });
      uint32_t stale = 0;
#pragma unroll
      for (int k = 0; k < kBlk; ++k)
        if (ov[k].y != tg) stale |= 1u << k;
      if (stale) repoll1(p, ov, stale, tg, [&](int k) { return pc + k * stride + e; });
      const float mk = __uint_as_float(ml[0].x), lk = __uint_as_float(ml[0].z);
      float Mb = fmaxf(M, mk);
#pragma unroll
      for (int o = 16; o; o >>= 1) Mb = fmaxf(Mb, __shfl_xor_sync(0xffffffffu, Mb, o));
      const float w = exp2_scale(mk, Mb);
      float lsum = lk * w;
#pragma unroll
      for (int o = 16; o; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
      const float r = exp2_scale(M, Mb);
      L = fmaf(L, r, lsum);
      acc *= r;
#pragma unroll
      for (int k = 0; k < kBlk; ++k) acc = fmaf(__uint_as_float(ov[k].x), __shfl_sync(0xffffffffu, w, k), acc);
      M = Mb;
    }
    // adjacent elements (lanes 2k, 2k + 1) go out as one bf16 pair
    const float o = acc / L, o_next = __shfl_down_sync(0xffffffffu, o, 1);
    if ((e & 1) == 0) st_word(p.attn_out + ((size_t)(h * G + g) * HD + e) / 2, bf2_word(o, o_next, tg));
  }
}

// Split-KV flash decoding of one (KV head, chunk) task on the tensor cores. The chunk's keys and
// values arrive in the ring as 128-byte-swizzled tiles (kv_off), so every ldmatrix below is free of
// bank conflicts. Per ring slot:
//   QK:  S = q K^T with mma.m16n8k16 (bf16 in, fp32 accumulate). The A operand holds the query heads
//        of this KV head's group in rows 0..G-1 and the bf16 residual of the same heads in rows
//        8..8+G-1, so q enters as hi + lo (~16 significant bits) while the keys stay exact bf16;
//        warps take 8-position tiles, write S to shared memory and their per-head maxima.
//   softmax: the slot maximum joins the running maximum M (log2 units: q is pre-scaled by
//        log2(e)/sqrt(hd)); P = 2^(S - M), split the same way into hi/lo rows of the P tile.
//   PV:  O += P V with mma.m16n8k16, warps over 8-dimension output tiles (and over position steps
//        when there are more warps than tiles); the running sum l comes from one more MMA against a
//        tile of ones, so l and O see the same P. O and l are rescaled by 2^(M_old - M) first.
// The chunk's (O, M, l) is written as its partial; the last chunk of the head to arrive merges them.
// The contraction is tiny (at most 4 query rows per KV head), so the legacy warp-level MMA serves:
// it replaces the per-lane FMA and shuffle work, which was the cost here, and needs no TMEM.
#ifndef AMK_INLINE_ATTN
#define AMK_INLINE_ATTN 0
#endif
template <int HD>
#if AMK_INLINE_ATTN
__device__ __forceinline__
#else
__device__ __noinline__
#endif
uint32_t attn_task(const Params& p, const Task t, uint32_t it, unsigned long long* tr) {
  const Smem s = smem_view();
  constexpr int NPS = kSlotBytes / (4 * HD);           // positions per ring slot (keys, then values)
  static_assert(NPS % 16 == 0, "a slot holds whole 16-row tensor boxes");
  static_assert(kMaxGroup * NPS * 4 + 2 * kMaxGroup * 4 + 16 * (NPS + 8) * 2 <= kAuxBytes,
                "scores, slot maxima and the P tile fit aux");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.Hq / p.Hkv;
  const int h = t.a, c = t.b, l = t.layer;
  const int P = p.pos + 1;
  const int C = attn_num_chunks(P, p.kv_block, attn_chunk_cap(P, p.kv_chunks_max, p.kv_chunks_short));
  if (c >= C) return it;
  int cb, ce;
  attn_chunk_range(P, C, c, &cb, &ce);

  if (p.sync && t.wait_ctr >= 0) wait_counter(p, t.wait_ctr, t.wait_mult);
  if (tr && tid == 0) tr[2] = globaltimer();

  // queries of this KV head's group, pre-scaled by log2(e) / sqrt(hd), as the A operand of the QK
  // MMAs (q tile: bf16 rows 0..G-1 the heads, rows 8..8+G-1 what rounding left over, other rows
  // zero), and this position's key and value rows (bf16), staged in shared memory (the GEMV
  // partial-sum region, which attention tasks do not use) in one round trip. The QKV stage publishes
  // them in packed row order: packed row j of a head is element j / 2 (j even) or hd/2 + j / 2 (j odd).
  const float qs = 1.4426950408889634f * rsqrtf((float)HD);
  constexpr int QSTR = HD * 2 + 16;                    // q tile row bytes (padded: conflict-free ldmatrix)
  uint8_t* const qtile = reinterpret_cast<uint8_t*>(s.part);
  uint16_t* kvc = reinterpret_cast<uint16_t*>(qtile + 16 * QSTR);   // [HD] k, then [HD] v
  static_assert(16 * QSTR + 4 * HD <= kPartBytes, "q tile and this position's k, v fit the partial region");
  auto unpack = [](int j) { return (j & 1) ? (j >> 1) + HD / 2 : (j >> 1); };
  for (int i = tid; i < 16 * QSTR / 16; i += kConsumerThreads) {   // rows past the group stay zero
    const int row = (i * 16) / QSTR;
    if ((row & 7) >= G) reinterpret_cast<uint4*>(qtile)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  {
    // up to two tagged pairs of q and (the first 2 * HD threads) one of k or v per thread, all in
    // one batch (G * HD <= 512)
    static_assert(kMaxGroup * 128 <= 2 * kConsumerThreads && 2 * 128 <= kConsumerThreads, "q, k, v pairs per thread");
    const uint32_t tg = tag_of(p.tag_epoch, l);
    const int ik = tid;
    const uint64_t* qa = p.qkv + (size_t)h * G * HD;
    const uint64_t* ka = p.qkv + (size_t)(p.Hq + (ik < HD ? 0 : p.Hkv) + h) * HD + (ik % HD);
    uint2 v[3] = {make_uint2(0u, tg), make_uint2(0u, tg), make_uint2(0u, tg)};
    if (tid < G * HD) v[0] = ld_pair(qa + tid);
    if (tid + kConsumerThreads < G * HD) v[1] = ld_pair(qa + tid + kConsumerThreads);
    if (ik < 2 * HD) v[2] = ld_pair(ka);
    const uint32_t stale = (v[0].y != tg ? 1u : 0u) | (v[1].y != tg ? 2u : 0u) | (v[2].y != tg ? 4u : 0u);
    if (stale) repoll1(p, v, stale, tg, [&](int j) { return j == 2 ? ka : qa + tid + j * kConsumerThreads; });
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int iq = tid + j * kConsumerThreads;
      if (iq < G * HD) {
        const float x = __uint_as_float(v[j].x) * qs;
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
        const int g = iq / HD, e = unpack(iq % HD);
        *reinterpret_cast<__nv_bfloat16*>(qtile + g * QSTR + 2 * e) = hi;
        *reinterpret_cast<__nv_bfloat16*>(qtile + (g + 8) * QSTR + 2 * e) = lo;
      }
    }
    if (ik < 2 * HD) kvc[(ik < HD ? 0 : HD) + unpack(ik % HD)] = f2bf(__uint_as_float(v[2].x));
  }
  float* const Ssm = s.aux;                                      // [kMaxGroup][NPS] scores
  int* const smax = reinterpret_cast<int*>(s.aux + kMaxGroup * NPS);   // [2][kMaxGroup] slot maxima (ordered keys)
  uint8_t* const ptile = reinterpret_cast<uint8_t*>(smax + 2 * kMaxGroup);
  constexpr int PSTR = (NPS + 8) * 2;                            // P tile row bytes (padded)
  // the P tile's rows past the group's heads stay zero for the whole task
  for (int i = tid; i < 16 * PSTR / 16; i += kConsumerThreads)
    reinterpret_cast<uint4*>(ptile)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (tid < 2 * kMaxGroup) smax[tid] = max_key(-CUDART_INF_F);
  bar_compute();
  if (tr && tid == 0) tr[10] = globaltimer();

  constexpr int KS = HD / 16;                          // k-steps of the QK contraction
  const int gid = lane >> 2, t4 = lane & 3;
  // this lane's row address in the q and P tiles for ldmatrix.x4 of an A operand (tile i of the four:
  // rows 8 (i & 1).., columns 8 (i >> 1).. of the 16-column step)
  const int arow = (((lane >> 3) & 1) << 3) | (lane & 7), acol = ((lane >> 4) & 1) << 3;
  const uint32_t qa_a = smem_u32(qtile) + arow * QSTR + acol * 2;

  // PV jobs: (output tile of 8 dimensions, position-step residue); most configurations give one
  // job per warp
  constexpr int NTO = HD / 8;
  constexpr int KSPLIT = kConsumerWarps / NTO > 1 ? kConsumerWarps / NTO : 1;
  constexpr int NJOBS = NTO * KSPLIT;
  constexpr int NJ = (NJOBS + kConsumerWarps - 1) / kConsumerWarps;
  float acc[NJ][4], lacc[NJ][4];
#pragma unroll
  for (int jb = 0; jb < NJ; ++jb)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[jb][i] = lacc[jb][i] = 0.f;
  float Mrun[kMaxGroup];
#pragma unroll
  for (int g = 0; g < kMaxGroup; ++g) Mrun[g] = -CUDART_INF_F;

  const uint32_t ptile_a = smem_u32(ptile);
  constexpr uint32_t kOnes = 0x3f803f80u;                        // bf16 pair (1, 1)

  for (int blk = cb, si = 0; blk < ce; blk += NPS, ++it, ++si) {
    const int slot = it % kSlots;
    wait_slot(p, &s.full[slot], (it / kSlots) & 1, (2u << 16) | slot);
    if (tr && tid == 0 && blk == cb) tr[11] = globaltimer();
    const int n = min(blk + NPS, ce) - blk;
    const int KT = (n + 15) >> 4;                       // 16-position steps
    uint8_t* const kb = s.ring + slot * kSlotBytes;
    uint8_t* const vb = kb + kSlotBytes / 2;
    const bool own = p.pos >= blk && p.pos < blk + n;
    if (own || (n & 15)) {
      // this step's own key/value row (the QK stage writes it in this launch) from the staged copy,
      // and zero value rows n..16 KT - 1 (loaded past the chunk: later positions may hold anything,
      // and P = 0 there must not meet a NaN); the proxy fence orders these generic writes before the
      // slot's next tensor copy
      constexpr int CH = HD / 8;                        // 16-byte chunks per row
      if (own && tid < 2 * CH) {
        const int jr = p.pos - blk, ch = tid % CH;
        uint8_t* dst = (tid < CH ? kb : vb) + kv_off(jr, ch, NPS);
        *reinterpret_cast<uint4*>(dst) = reinterpret_cast<const uint4*>(kvc + (tid < CH ? 0 : HD))[ch];
      }
      for (int i = tid; i < (16 * KT - n) * CH; i += kConsumerThreads)
        *reinterpret_cast<uint4*>(vb + kv_off(n + i / CH, i % CH, NPS)) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      bar_compute();
    }
    // ---- QK: warps over 8-position tiles ----
    const int NT = (n + 7) >> 3;
    float wm = -CUDART_INF_F;
    const uint32_t kb_a = smem_u32(kb);
    int* const mx = smax + (si & 1) * kMaxGroup;
    if (warp < NT) {
      // the q fragments, for this slot's tiles of the warp (not held across the slot: registers)
      uint32_t qf[KS][4];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) ldsm_x4(qf[ks], qa_a + 32 * ks);
      for (int nt = warp; nt < NT; nt += kConsumerWarps) {
        // two accumulator chains (even and odd k-steps): half the dependent MMA latency
        float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
        const int r = nt * 8 + (lane & 7);
        uint32_t b[KS / 2][4];
#pragma unroll
        for (int kk = 0; kk < KS / 2; ++kk) ldsm_x4(b[kk], kb_a + kv_off(r, 4 * kk + (lane >> 3), NPS));
#pragma unroll
        for (int kk = 0; kk < KS / 2; ++kk) {
          mma_bf16_16816(d, qf[2 * kk], b[kk][0], b[kk][1]);
          mma_bf16_16816(e, qf[2 * kk + 1], b[kk][2], b[kk][3]);
        }
        const int j0 = nt * 8 + 2 * t4;
        const float s0 = j0 < n ? (d[0] + e[0]) + (d[2] + e[2]) : -CUDART_INF_F;
        const float s1 = j0 + 1 < n ? (d[1] + e[1]) + (d[3] + e[3]) : -CUDART_INF_F;
        if (gid < G) *reinterpret_cast<float2*>(Ssm + gid * NPS + j0) = make_float2(s0, s1);
        wm = fmaxf(wm, fmaxf(s0, s1));
      }
    }
    wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, 1));
    wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, 2));
    if (gid < G && t4 == 0 && warp < NT) atomicMax(mx + gid, max_key(wm));
    bar_compute();
    // ---- the new running maxima (every thread, identically) from the slot maxima; the other buffer
    //      is reset for the next slot ----
    float Mnew[kMaxGroup], alpha[kMaxGroup];
    {
      static_assert(kMaxGroup == 4, "one 16-byte read of the slot maxima");
      const int4 k4 = *reinterpret_cast<const int4*>(mx);
      const float ms[kMaxGroup] = {key_max(k4.x), key_max(k4.y), key_max(k4.z), key_max(k4.w)};
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) {
        Mnew[g] = fmaxf(Mrun[g], ms[g]);
        alpha[g] = exp2_scale(Mrun[g], Mnew[g]);
        Mrun[g] = Mnew[g];
      }
      if (tid < kMaxGroup) smax[((si + 1) & 1) * kMaxGroup + tid] = max_key(-CUDART_INF_F);
    }
    // ---- P = 2^(S - M) as hi/lo bf16 rows of the P tile, two positions per thread ----
    {
      const int W2 = 8 * KT;                            // position pairs per head (16 KT positions)
      for (int e = tid; e < G * W2; e += kConsumerThreads) {
        const int g = e / W2, j = 2 * (e % W2);
        const float M = g == 0 ? Mnew[0] : g == 1 ? Mnew[1] : g == 2 ? Mnew[2] : Mnew[3];
        const float p0 = j < n ? fast_exp2(Ssm[g * NPS + j] - M) : 0.f;
        const float p1 = j + 1 < n ? fast_exp2(Ssm[g * NPS + j + 1] - M) : 0.f;
        uint32_t hi, lo;
        split_bf2(p0, p1, hi, lo);
        *reinterpret_cast<uint32_t*>(ptile + g * PSTR + j * 2) = hi;
        *reinterpret_cast<uint32_t*>(ptile + (g + 8) * PSTR + j * 2) = lo;
      }
    }
    bar_compute();
    // ---- PV ----
    const float al = gid == 0 ? alpha[0] : gid == 1 ? alpha[1] : gid == 2 ? alpha[2] : gid == 3 ? alpha[3] : 1.f;
    const uint32_t vb_a = smem_u32(vb);
#pragma unroll
    for (int jb = 0; jb < NJ; ++jb) {
      const int job = warp + jb * kConsumerWarps;
      if (job < NJOBS) {
        const int ntile = job % NTO, kpart = job / NTO;
#pragma unroll
        for (int i = 0; i < 4; ++i) { acc[jb][i] *= al; lacc[jb][i] *= al; }
        // two position steps per round, their operands loaded first and accumulated in separate
        // registers (added at the end of the slot): half the dependent MMA latency
        const uint32_t pa = ptile_a + arow * PSTR + acol * 2;
        const int vr = arow;   // ldmatrix.x2.trans: lanes 0..15 give rows 0..15 of the position step
        float a2[4] = {0.f, 0.f, 0.f, 0.f}, l2[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ks = kpart; ks < KT; ks += 2 * KSPLIT) {
          const bool two = ks + KSPLIT < KT;
          uint32_t a[4], c[4] = {0u, 0u, 0u, 0u}, b0, b1, b2 = 0u, b3 = 0u;
          ldsm_x4(a, pa + 32 * ks);
          ldsm_x2_trans(b0, b1, vb_a + kv_off(16 * ks + vr, ntile, NPS));
          if (two) {
            ldsm_x4(c, pa + 32 * (ks + KSPLIT));
            ldsm_x2_trans(b2, b3, vb_a + kv_off(16 * (ks + KSPLIT) + vr, ntile, NPS));
          }
          mma_bf16_16816(acc[jb], a, b0, b1);
          if (ntile == 0) mma_bf16_16816(lacc[jb], a, kOnes, kOnes);
          if (two) {
            mma_bf16_16816(a2, c, b2, b3);
            if (ntile == 0) mma_bf16_16816(l2, c, kOnes, kOnes);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) { acc[jb][i] += a2[i]; lacc[jb][i] += l2[i]; }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[slot]);
  }

  if (tr && tid == 0) tr[4] = globaltimer();
  // ---- the chunk's partial: O (unnormalised), M and l per query head ----
  if constexpr (KSPLIT > 1) {
    // jobs of the later position residues hand their accumulators to residue 0 through the P tile
    float* xs = reinterpret_cast<float*>(ptile);
    bar_compute();
#pragma unroll
    for (int jb = 0; jb < NJ; ++jb) {
      const int job = warp + jb * kConsumerWarps;
      const int ntile = job % NTO, kpart = job / NTO;
      if (job < NJOBS && kpart > 0) {
        float* e = xs + (((kpart - 1) * NTO + ntile) * 32 + lane) * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) { e[i] = acc[jb][i]; e[4 + i] = lacc[jb][i]; }
      }
    }
    bar_compute();
#pragma unroll
    for (int jb = 0; jb < NJ; ++jb) {
      const int job = warp + jb * kConsumerWarps;
      const int ntile = job % NTO, kpart = job / NTO;
      if (job < NJOBS && kpart == 0) {
        for (int k = 1; k < KSPLIT; ++k) {
          const float* e = xs + (((k - 1) * NTO + ntile) * 32 + lane) * 8;
#pragma unroll
          for (int i = 0; i < 4; ++i) { acc[jb][i] += e[i]; lacc[jb][i] += e[4 + i]; }
        }
      }
    }
  }
  {
    const uint32_t tg = tag_of(p.tag_epoch, l);
#pragma unroll
    for (int jb = 0; jb < NJ; ++jb) {
      const int job = warp + jb * kConsumerWarps;
      const int ntile = job % NTO, kpart = job / NTO;
      if (job < NJOBS && kpart == 0 && gid < G) {
        uint64_t* dg = p.attn_part + (((size_t)h * G + gid) * p.kv_chunks_max + c) * (HD + 2);
        st_pair2(dg + ntile * 8 + 2 * t4, acc[jb][0] + acc[jb][2], acc[jb][1] + acc[jb][3], tg);
        if (ntile == 0 && t4 == 0) {
          const float M = gid == 0 ? Mrun[0] : gid == 1 ? Mrun[1] : gid == 2 ? Mrun[2] : Mrun[3];
          st_pair2(dg + HD, M, lacc[jb][0] + lacc[jb][2], tg);   // (hd + 2) even: 16-byte aligned
        }
      }
    }
  }
  if (tr && tid == 0) tr[5] = globaltimer();
  if (!p.sync) return it;
  // ticket: the last chunk of this head to arrive merges all of them and signals. A relaxed atomic:
  // the merge checks the tags of every partial it reads.
  bar_compute();
  uint32_t* ticket = p.attn_ticket + l * p.Hkv + h;
  if (tid == 0) s.misc->flag = (atom_relaxed_add(ticket, 1u) == (uint32_t)(C - 1));
  bar_compute();
  if (tr && tid == 0) tr[6] = globaltimer();
  if (s.misc->flag) {
    merge_head<HD>(p, h, C, l);
    bar_compute();
    if (tid == 0) {
      *ticket = 0u;
      red_relaxed_add(p.ctr + t.sig_ctr, 1u);
    }
    if (tr && tid == 0) tr[7] = globaltimer();
  }
  bar_compute();
  return it;
}

// ------------------------------------------------------------------------------------------------
// Grid argmax of the per-CTA LM maxima (lowest index on ties). Called by all compute threads.

__device__ __noinline__ void grid_argmax(const Params& p) {
  const Smem s = smem_view();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float bv = -CUDART_INF_F;
  int bi = 0x7fffffff;
  const uint32_t tg = tag_of(p.tag_epoch, p.L);
  for (int b = threadIdx.x; b < p.grid; b += kConsumerThreads) {
    // {max, index} as two tagged pairs: re-read until both tags are this launch's (bounded)
    uint4 e[1] = {ld_pair2(p.am + 2 * b)};
    if (!tags_ok(e[0], tg)) repoll2(p, e, 1u, tg, [&](int) { return p.am + 2 * b; });
    const float v = __uint_as_float(e[0].x);
    const int i = (int)e[0].z;
    if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
  }
  if (lane == 0) { s.misc->am_v[warp] = bv; s.misc->am_i[warp] = bi; }
  bar_compute();
  if (threadIdx.x == 0) {
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float ov = s.misc->am_v[w];
      const int oi = s.misc->am_i[w];
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    *p.next_token = (bi >= 0 && bi < p.V) ? bi : -1;
  }
  bar_compute();
}

// ------------------------------------------------------------------------------------------------
// Compute warps

__device__ void compute(const Params& p, const Task* tasks, int nt) {
  const Smem s = smem_view();
  const int tid = threadIdx.x;
  if (tid == 0) {
    int tok = p.token;
    if (tok < 0) tok = __ldcg(p.next_token);
    if (tok < 0 || tok >= p.V) {
      raise_abort(p, (4u << 16));
      tok = 0;
    }
    s.misc->token = tok;
    s.misc->lm_v = -CUDART_INF_F;
    s.misc->lm_i = 0x7fffffff;
  }
  bar_compute();
  const int token = s.misc->token;
  uint32_t it = 0;
  for (int ti = 0; ti < nt; ++ti) {
    const Task t = tasks[ti];
    unsigned long long* tr = p.trace ? p.trace + ((size_t)blockIdx.x * p.max_tasks_per_cta + ti) * AMK_TRACE_WORDS : nullptr;
    if (tr && tid == 0) {
      tr[0] = ((unsigned long long)t.op << 32) | (unsigned long long)t.layer << 16 | (unsigned)ti;
      tr[1] = tr[2] = globaltimer();
      tr[13] = clock64();
    }
    if (is_gemv(t.op)) {
      const GemvGeom& g = p.geom[gemv_slot_of(t.op)];
      const int wk = t.op == OP_LM && p.tied ? AMK_W_BF16 : p.wdtype;   // a tied head reads the bf16 table
      if (wk == AMK_W_INT8) {
        switch (g.gb) {
          case 32:
#if AMK_INLINE_HOT
            if (g.nr <= 1) { it = gemv_body<1, 32, 1>(p, t, it, token, tr); break; }
#endif
            it = gemv_nr<1, 32>(p, t, it, token, tr, g.nr); break;
          case 16: it = gemv_nr<1, 16>(p, t, it, token, tr, g.nr); break;
          case 8: it = gemv_nr<1, 8>(p, t, it, token, tr, g.nr); break;
          case 4: it = gemv_nr<1, 4>(p, t, it, token, tr, g.nr); break;
          default: it = gemv_nr<1, 2>(p, t, it, token, tr, g.nr); break;
        }
      } else if (wk == AMK_W_INT4) {
        switch (g.gb) {
#if AMK_I4_MAX_GB >= 32
          case 32: it = gemv_nr<2, 32>(p, t, it, token, tr, g.nr); break;
#endif
          case 16:
#if AMK_INLINE_HOT4
            if (g.nr <= 1 && g.rb % (32 * 16) == 0) { it = gemv_body<2, 16, 1, false>(p, t, it, token, tr); break; }
#endif
            it = gemv_nr<2, 16>(p, t, it, token, tr, g.nr); break;
          case 8: it = gemv_nr<2, 8>(p, t, it, token, tr, g.nr); break;
          default: it = gemv_nr<2, 4>(p, t, it, token, tr, g.nr); break;
        }
      } else {
        switch (g.gb) {
          case 64: it = gemv_nr<0, 64>(p, t, it, token, tr, g.nr); break;
          case 32: it = gemv_nr<0, 32>(p, t, it, token, tr, g.nr); break;
          case 16: it = gemv_nr<0, 16>(p, t, it, token, tr, g.nr); break;
          case 8: it = gemv_nr<0, 8>(p, t, it, token, tr, g.nr); break;
          default: it = gemv_nr<0, 4>(p, t, it, token, tr, g.nr); break;
        }
      }
      if (t.op == OP_LM) {
        if (t.flags & kLastOfStage) {
          // this CTA's maximum as one tagged 16-byte store; the last CTA to take the ticket reduces
          // them all, re-reading any entry whose tags are not this launch's yet (no fence needed)
          if (tid == 0)
            st_pair2(p.am + 2 * blockIdx.x, s.misc->lm_v, __int_as_float(s.misc->lm_i), tag_of(p.tag_epoch, p.L));
          if (p.sync) {
            bar_compute();
            if (tid == 0) s.misc->flag = (atom_relaxed_add(p.am_ticket, 1u) == (uint32_t)(p.grid - 1));
            bar_compute();
            if (s.misc->flag) {
              grid_argmax(p);
              if (tid == 0) *p.am_ticket = 0u;
            }
          }
        }
      } else if (p.sync && (t.flags & kLastOfStage) && t.sig_ctr >= 0) {
        bar_compute();
        signal_counter(p, t.sig_ctr);
      }
      if (tr && tid == 0) tr[7] = globaltimer();
    } else if (t.op == OP_ATTN) {
      if (p.hd == 64) it = attn_task<64>(p, t, it, tr);
      else it = attn_task<128>(p, t, it, tr);
    } else if (t.op == OP_MERGE) {
      const int C = attn_num_chunks(p.pos + 1, p.kv_block, attn_chunk_cap(p.pos + 1, p.kv_chunks_max, p.kv_chunks_short));
      if (p.hd == 64) merge_head<64>(p, t.a, C, t.layer);
      else merge_head<128>(p, t.a, C, t.layer);
    } else if (t.op == OP_ARGMAX) {
      grid_argmax(p);
    }
    if (tr && tid == 0) {
      tr[3] = globaltimer();
      tr[14] = clock64();
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params p) {
  Smem s = carve(smem_raw);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kConsumerWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
  }
  // this CTA's task list into shared memory when it fits (read at every task boundary by the
  // producer and the compute warps; a global read there is an L2 round trip on the critical path)
  const int b = blockIdx.x;
  const Task* tasks = p.tasks + p.task_off[b];
  const int nt = p.task_off[b + 1] - p.task_off[b];
  if (p.sync && nt <= kTaskCache) {   // the op-per-kernel launches read one or two tasks each
    Task* cache = reinterpret_cast<Task*>(smem_raw + kSmemBytes - kTaskCacheBytes);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(tasks);
    uint32_t* dst = reinterpret_cast<uint32_t*>(cache);
    for (int i = threadIdx.x; i < nt * (int)(sizeof(Task) / 4); i += kThreads) dst[i] = __ldg(src + i);
    tasks = cache;
  }
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) {
    if (threadIdx.x == kConsumerThreads) producer(p, tasks, nt);
    return;
  }
  compute(p, tasks, nt);
}

// ------------------------------------------------------------------------------------------------
// Weight packer: one CTA per packed row.

__global__ void pack_kernel(int role, int hd, int ffn, const void* src, int src_dtype, int cols, int dst_dtype,
                            void* dst, uint16_t* scales) {
  __shared__ float red[32];
  const int pr = blockIdx.x;
  const int sr = packed_row_source(role, hd, ffn, pr);
  auto load = [&](int k) -> float {
    if (src_dtype == AMK_SRC_F32) return static_cast<const float*>(src)[(size_t)sr * cols + k];
    return bf2f(static_cast<const uint16_t*>(src)[(size_t)sr * cols + k]);
  };
  if (dst_dtype == AMK_W_BF16) {
    uint16_t* out = static_cast<uint16_t*>(dst) + (size_t)pr * cols;
    for (int k = threadIdx.x; k < cols; k += blockDim.x) out[k] = f2bf(load(k));
    return;
  }
  float amax = 0.f;
  for (int k = threadIdx.x; k < cols; k += blockDim.x) amax = fmaxf(amax, fabsf(load(k)));
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (threadIdx.x == 0) red[0] = a;
  }
  __syncthreads();
  const float qmax = dst_dtype == AMK_W_INT4 ? 7.f : 127.f;
  const uint16_t sb = f2bf(__fdiv_rn(red[0], qmax));
  const float s = bf2f(sb);
  if (threadIdx.x == 0) scales[pr] = sb;
  auto quant = [&](int k) -> int {
    float q = 0.f;
    if (s > 0.f) q = fminf(qmax, fmaxf(-qmax, rintf(__fdiv_rn(load(k), s))));
    return (int)q;
  };
  if (dst_dtype == AMK_W_INT4) {   // byte j: element 2j in the low nibble, 2j + 1 in the high, each + 8
    uint8_t* out = static_cast<uint8_t*>(dst) + (size_t)pr * (cols / 2);
    for (int j = threadIdx.x; j < cols / 2; j += blockDim.x)
      out[j] = (uint8_t)((quant(2 * j) + 8) | ((quant(2 * j + 1) + 8) << 4));
    return;
  }
  int8_t* out = static_cast<int8_t*>(dst) + (size_t)pr * cols;
  for (int k = threadIdx.x; k < cols; k += blockDim.x) out[k] = (int8_t)quant(k);
}

}  // namespace dev

// ------------------------------------------------------------------------------------------------
// Host-side launch helpers (called from amk_api.cu)

cudaError_t prepare_kernel_attributes() {
  return cudaFuncSetAttribute(dev::decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
}

cudaError_t occupancy(int* blocks_per_sm) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, dev::decode_kernel, kThreads, kSmemBytes);
}

cudaError_t launch_decode(const Params& p, cudaStream_t stream, bool cooperative) {
  void* args[] = {const_cast<Params*>(&p)};
  if (cooperative)
    return cudaLaunchCooperativeKernel((const void*)dev::decode_kernel, dim3(p.grid), dim3(kThreads), args, kSmemBytes,
                                       stream);
  return cudaLaunchKernel((const void*)dev::decode_kernel, dim3(p.grid), dim3(kThreads), args, kSmemBytes, stream);
}

cudaError_t launch_pack(int role, int hd, int ffn, const void* src, int src_dtype, int rows, int cols, int dst_dtype,
                        void* dst, void* scales, cudaStream_t stream) {
  dev::pack_kernel<<<rows, 256, 0, stream>>>(role, hd, ffn, src, src_dtype, cols, dst_dtype, dst,
                                             static_cast<uint16_t*>(scales));
  return cudaGetLastError();
}

}  // namespace amk
