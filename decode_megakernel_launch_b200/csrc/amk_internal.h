// Internal layout shared by the host planner, the host API and the device code of libamk.
//
// The persistent kernel follows the Layer-0 design of "AutoMegaKernel: A Statically-Checked Agent
// Harness for Self-Retargeting Megakernel Synthesis" (technical summary, "Methodology"): one CTA per
// SM walks its own task list in a globally valid order, each task doing wait -> dispatch -> signal
// on monotonic counters. Here the task list is a fixed per-layer pattern built on the host:
//   per layer l:  QKV(l) -> ATTN(l) -> O(l) -> GU(l) -> DOWN(l);   then LM (head + argmax).
// Every GEMV stage is row-split over all CTAs; ATTN is split over (KV head, KV chunk).
#pragma once
#include <cuda.h>       // CUtensorMap (the descriptors are encoded through the runtime's driver entry point)
#include <stdint.h>

#include "../../include/amk.h"

#ifdef __CUDACC__
#define AMK_HD __host__ __device__
#else
#define AMK_HD
#endif

namespace amk {

// ---- CTA shape and shared-memory budget ------------------------------------------------------
// Compute warps (a compile-time knob). With the producer, 17 warps put 5 on one SM sub-partition,
// which caps every thread at 96 registers; 15 + 1 would leave 128.
#ifndef AMK_CONSUMER_WARPS
#define AMK_CONSUMER_WARPS 16
#endif
constexpr int kConsumerWarps   = AMK_CONSUMER_WARPS;
constexpr int kConsumerThreads = kConsumerWarps * 32;      // compute threads
constexpr int kThreads         = kConsumerThreads + 32;    // + 1 producer (bulk-copy) warp
// Ring geometry (compile-time; -DAMK_SLOT_BYTES / -DAMK_SLOTS / -DAMK_INFLIGHT override it).
// kInflight bounds the copies the producer keeps outstanding: every other global access of the SM
// queues behind them, so fewer bytes in flight than the ring holds keeps those accesses short
// while a stalled consumer still lets the ring fill to kSlots ahead.
#ifndef AMK_SLOT_BYTES
#define AMK_SLOT_BYTES 65536
#endif
#ifndef AMK_SLOTS
#define AMK_SLOTS 3
#endif
#ifndef AMK_INFLIGHT
#define AMK_INFLIGHT 1
#endif
constexpr int kSlotBytes       = AMK_SLOT_BYTES;           // one bulk-copy ring slot
constexpr int kSlots           = AMK_SLOTS;                // ring depth
constexpr int kInflight        = AMK_INFLIGHT;             // outstanding copies, <= kSlots
// The producer warms L2 with up to kPfItems upcoming ring items, one per kPfGapNs (a little faster
// than one SM's share of HBM bandwidth: 64 KB per 1.2 us on 148 SMs is 7.9 TB/s; at 0.8 us the
// queues it builds slow every other load), so HBM keeps streaming through the stage transitions:
// while the compute warps hold a landed slot longer than kStallNs (they wait on a counter) and,
// with kPfContinuous, between stalls too. 10 items of 64 KB on 148 SMs use at most 97 MB of the
// 126 MB L2. kPfItems = 0 disables it.
#ifndef AMK_PF_ITEMS
#define AMK_PF_ITEMS 10
#endif
#ifndef AMK_PF_GAP_NS
#define AMK_PF_GAP_NS 1200
#endif
#ifndef AMK_PF_CONTINUOUS
#define AMK_PF_CONTINUOUS 1
#endif
#ifndef AMK_PF_STALL_NS
#define AMK_PF_STALL_NS 200
#endif
constexpr int kPfItems = AMK_PF_ITEMS;
constexpr unsigned kPfGapNs = AMK_PF_GAP_NS;
constexpr unsigned kStallNs = AMK_PF_STALL_NS;
constexpr bool kPfContinuous = AMK_PF_CONTINUOUS != 0;
static_assert(kInflight >= 1 && kInflight <= kSlots, "ring in-flight bound");
static_assert(kSlotBytes % 256 == 0 && kSlotBytes >= 32768, "ring slot holds a 32 KB weight row");
constexpr int kRowBlock        = 128;                      // GEMV rows per epilogue block
constexpr int kMaxTaskRows     = kConsumerThreads * 2 >= 1024 ? 1024 : kConsumerThreads * 2;   // rows of one GEMV task
// Rows per register batch of the GEMV inner loop for 64- and 32-byte groups (the transposed
// butterfly reduces 2 or 4 rows at once).
#ifndef AMK_NB64
#define AMK_NB64 1
#endif
#ifndef AMK_NB32
#define AMK_NB32 4
#endif
// Largest int4 group (bytes of nibbles per thread per row): 16 B = 32 elements, 32 B = 64.
#ifndef AMK_I4_MAX_GB
#define AMK_I4_MAX_GB 16
#endif
// The hot GEMV instances (int8 with 32-byte groups, int4 with 16-byte groups, one group per thread)
// inlined into the kernel's task loop (1) or called (0).
#ifndef AMK_INLINE_HOT
#define AMK_INLINE_HOT 1
#endif
#ifndef AMK_INLINE_HOT4
#define AMK_INLINE_HOT4 1
#endif
// int4 high nibbles: masked in place and met with an unsigned-byte dp2a (1) or shifted down (0).
#ifndef AMK_I4_NOSHIFT
#define AMK_I4_NOSHIFT 1
#endif
constexpr int kMaxGroup        = 4;                        // Hq / Hkv supported
constexpr int kAuxBytes        = 8 * kMaxGroup * (128 + 2) * 4;   // attention cross-warp tree
constexpr int kRingBytes       = kSlots * kSlotBytes;
constexpr int kPartBytes       = kConsumerWarps * kRowBlock * 4;
constexpr int kScaleBytes      = kMaxTaskRows * 4;
constexpr int kMiscBytes       = 512;
constexpr int kTaskCache       = 192;                      // task list copied to shared memory when it fits
constexpr int kTaskCacheBytes  = kTaskCache * 32;
constexpr int kSmemBytes       = kRingBytes + kPartBytes + kAuxBytes + kScaleBytes + kMiscBytes + kTaskCacheBytes;
static_assert(kSmemBytes <= 227 * 1024, "dynamic shared memory of one CTA");
static_assert(kAuxBytes >= kMaxTaskRows * 4 && kAuxBytes >= 128 * 4, "aux holds a GEMV task's residual rows or a RoPE row");

// ---- tagged activations ----------------------------------------------------------------------
// Every vector one CTA hands to others travels in 64-bit tagged words, each one aligned 8-byte
// element of the store that writes it and of the load that reads it, so a reader that sees the tag
// sees the payload: the high word is the tag, the low word either two bf16 values (the GEMV inputs:
// x after O and after down, the merged attention, the SwiGLU output; the 16-bit activations of
// W8A16) or one fp32 value (the packed q / k / v rows, the attention partials, the LM-head maxima).
// A reader accepts a word only when its tag is the one it expects and re-reads the others, so the
// writer needs no release fence (under the full weight stream a gpu-scope fence costs several
// microseconds: it waits on the SM's in-flight weight copies); the stage counters, bumped with
// relaxed reductions, only tell readers of a wide vector when to start reading it. The residual
// stream itself stays fp32: each CTA keeps its own rows of x (O and down split rows the same way).
// The tag names the launch, the layer and (for x) the version: tag = epoch * 2048 + 2 * layer + k,
// k = 0 for x after O and for every other vector, 1 for x after down.
AMK_HD inline uint32_t tag_of(uint32_t epoch, int layer, int k = 0) { return epoch * 2048u + 2u * (uint32_t)layer + (uint32_t)k; }
constexpr int kMaxLayers = 1023;   // 2 * layer + 1 < 2048, the LM head's entries use layer = n_layers

// ---- tasks -----------------------------------------------------------------------------------
enum Op : uint16_t {
  OP_QKV = 1,     // RMSNorm(x)*g1 -> packed QKV GEMV -> RoPE -> q scratch, K/V cache at pos
  OP_ATTN = 2,    // GQA attention of one KV head over one KV chunk -> partial (m, l, o)
  OP_O = 3,       // O GEMV + residual into x
  OP_GU = 4,      // RMSNorm(x)*g2 -> gate/up GEMV -> SwiGLU -> act scratch
  OP_DOWN = 5,    // down GEMV + residual into x
  OP_LM = 6,      // RMSNorm(x)*gf -> LM-head GEMV -> logits + per-CTA argmax
  OP_MERGE = 7,   // (op-per-kernel ablation only) log-sum-exp merge of one KV head's partials
  OP_ARGMAX = 8,  // (op-per-kernel ablation only) grid argmax of the per-CTA maxima
};

// GEMV op index into Params::geom
AMK_HD inline int gemv_slot_of(int op) {
  return op == OP_QKV ? 0 : op == OP_O ? 1 : op == OP_GU ? 2 : op == OP_DOWN ? 3 : 4;
}

// Counters: per layer one per stage kind, then nothing else (the argmax and the attention merge
// use tickets, which the last arriver resets).
enum CtrKind { CTR_QKV = 0, CTR_ATTN = 1, CTR_O = 2, CTR_GU = 3, CTR_DOWN = 4, CTR_PER_LAYER = 5 };

struct Task {
  uint16_t op;
  uint16_t layer;
  int32_t  a;          // GEMV: first packed row;  ATTN: KV head;  MERGE: KV head
  int32_t  b;          // GEMV: number of rows;    ATTN: chunk index
  int32_t  wait_ctr;   // counter to wait on, -1 = none
  uint32_t wait_mult;  // wait until counter >= epoch * wait_mult (mod 2^32)
  int32_t  sig_ctr;    // counter to add 1 to when done, -1 = none
  uint32_t flags;      // kFirstOfStage | kLastOfStage: only the first task of a stage on a CTA
                       // waits, only the last signals (a stage split into several tasks on one
                       // CTA still signals once)
  uint32_t pad;
};
constexpr uint32_t kFirstOfStage = 1u;
constexpr uint32_t kLastOfStage = 2u;
constexpr uint32_t kTagWait = 4u;      // no counter: the task polls the tags of its (small) inputs

// How one GEMV shape maps onto the compute threads. A row of `rb` bytes is cut into groups of
// `gb` bytes (one shared-memory vector load per thread); `wg_total` warps' worth of groups cover a
// row (the lanes of the last warp past the row's end stay idle). Warps form `rp` row groups of `wpg` warps; a thread keeps the activations of its groups in
// registers for the whole task (`nr` groups per thread).
struct GemvGeom {
  int32_t K;         // elements per row
  int32_t rb;        // bytes per row
  int32_t gb;        // bytes per group: 64, 32, 16, 8, 4 or 2
  int32_t wg_total;  // ceil((rb / gb) / 32): warps of groups per row (the last one may be partly filled)
  int32_t wpg;       // warps per row group
  int32_t nr;        // groups per thread
  int32_t rp;        // row groups
  int32_t rs;        // rows per ring slot
};

struct LayerPtrs {
  const void*     wqkv;
  const void*     wo;
  const void*     wgu;
  const void*     wdown;
  const uint16_t* sqkv;
  const uint16_t* so;
  const uint16_t* sgu;
  const uint16_t* sdown;
  const uint16_t* attn_norm;
  const uint16_t* ffn_norm;
};

struct Params {
  // model
  int L, d, Hq, Hkv, hd, ffn, V, max_seq;
  float eps;
  int wdtype;          // AMK_W_INT8 / AMK_W_BF16 / AMK_W_INT4
  int tied;
  int grid;
  const LayerPtrs* layers;     // device [L]
  const uint16_t* embed;       // bf16 [V, d]
  const uint16_t* final_norm;  // bf16 [d]
  const void*     lm_w;        // packed head or the embedding when tied
  const uint16_t* lm_s;        // scales or null
  uint16_t* kcache;            // bf16 [L][Hkv][max_seq][hd]
  uint16_t* vcache;
  // the caches as 2-D [L Hkv max_seq][hd] bf16 tensors with 128-byte swizzle: [0] boxes of 64
  // columns x 64 rows, [1] of 64 columns x 16 rows (for the last rows of a chunk)
  CUtensorMap kmap[2], vmap[2];
  const float* rope;           // interleaved (cos, sin) [max_seq][hd/2][2]
  // scratch (device)
  // tagged words (see tag_of)
  uint64_t* x;                 // x as bf16 pairs [d / 2] (after O, then after down)
  float* xres;                 // x in fp32 [d]: each CTA reads back only the rows it wrote
  uint64_t* qkv;               // QKV outputs in packed row order [(Hq + 2 Hkv) hd], fp32: roped q, roped k
                               //   and v rounded to bf16 (this position's keys and values, as cached)
  uint64_t* attn_out;          // merged attention as bf16 pairs [Hq * hd / 2]
  uint64_t* act;               // SwiGLU output as bf16 pairs [ffn / 2]
  uint64_t* attn_part;         // [Hkv][G][kv_chunks_max][hd + 2], fp32: o, then m and l of each chunk
  uint64_t* am;                // [grid][2] LM-head maximum and its index
  uint32_t* ctr;               // [L * CTR_PER_LAYER]
  uint32_t* attn_ticket;       // [L * Hkv]
  uint32_t* am_ticket;         // [1]
  uint32_t* abort_flag;        // device word: nonzero after a wait expired
  volatile uint32_t* status;   // host-mapped sticky status word
  unsigned long long* trace;   // [grid][max_tasks_per_cta][4] or null
  int max_tasks_per_cta;
  // plan
  const Task* tasks;           // this launch's task list
  const int*  task_off;        // [grid + 1]
  GemvGeom geom[5];            // QKV, O, GU, DOWN, LM
  int kv_block;
  int kv_chunks_max;           // attention chunks per KV head at most (the plan's tasks, partial rows)
  int kv_chunks_short;         // the cap below kLongContext positions
  unsigned long long timeout_ns;
  // per launch
  uint32_t epoch;              // counter targets are epoch * producers
  uint32_t tag_epoch;          // tags of this launch's vectors (tag_of)
  int token;                   // >= 0, or -1 to read *next_token
  int pos;
  float* logits;               // may be null
  int*   next_token;
  int sync;                    // 1 = persistent megakernel (waits/signals), 0 = op-per-kernel
};

// Encodes p.kmap and p.vmap from p.kcache, p.vcache and the dims in p (host). Returns AMK_OK or
// AMK_ERR_CUDA when the driver's encoder is unavailable or refuses the layout.
int encode_kv_maps(Params& p);

// ---- shared host/device helpers ----------------------------------------------------------------
AMK_HD inline int packed_row_source(int role, int hd, int ffn, int packed_row) {
  if (role == AMK_ROLE_QKV) {
    int head = packed_row / hd, j = packed_row % hd;
    return head * hd + ((j & 1) ? (j >> 1) + hd / 2 : (j >> 1));
  }
  if (role == AMK_ROLE_GATE_UP) return (packed_row & 1) ? ffn + (packed_row >> 1) : (packed_row >> 1);
  return packed_row;
}

// Attention chunking of positions 0..P-1 of one KV head: chunks of cs = ceil(P / c) positions,
// c = min(cmax, ceil(P / kv_block)); the count returned is ceil(P / cs), so no chunk is empty.
// Chunk cap for P positions: below kLongContext the merge's one 16-chunk batch (one L2 round trip)
// beats spreading a short cache over every CTA; from there on each chunk streams several ring slots
// and more CTAs pay more (1B-shaped, 32K positions: 16 chunks 0.930 ms, 18 chunks 0.913 ms per step;
// 8B-shaped, 1K: 16 chunks 1.850 ms, 18 chunks 1.877 ms).
constexpr int kLongContext = 4096;
AMK_HD inline int attn_chunk_cap(int P, int cmax, int cshort) { return P >= kLongContext ? cmax : cshort; }
AMK_HD inline int attn_num_chunks(int P, int kv_block, int cmax) {
  if (P < 1) return 1;
  int c = (P + kv_block - 1) / kv_block;
  if (c > cmax) c = cmax;
  if (c < 1) c = 1;
  int cs = (P + c - 1) / c;
  return (P + cs - 1) / cs;
}
AMK_HD inline void attn_chunk_range(int P, int C, int c, int* begin, int* end) {
  int cs = (P + C - 1) / C;
  int b = c * cs, e = b + cs;
  if (b > P) b = P;
  if (e > P) e = P;
  *begin = b;
  *end = e;
}
AMK_HD inline int attn_positions_per_slot(int hd) { return kSlotBytes / (2 * hd * 2); }

}  // namespace amk
