// groups.cuh -- layout of a token grouping (the caller's buffer built by
// group_plan_kernel in grouped.cu), shared by the kernels that read it: the
// grouped combine (grouped.cu) and the training step (train.cu).
#pragma once

#include "combine_common.cuh"

namespace mole {
namespace {

constexpr int kItemTokens = 16;     // tokens per work item

// Per-CTA totals of step 1: [0] tokens, [n] work items of n tokens (n =
// 1..kItemTokens), [kAgg] distinct ids.
constexpr int kAgg = kItemTokens + 1;

// Control words (set to 0xFFFFFFFF when a grouping is built): work items,
// the three grid-barrier counters, the abort word, the running totals of
// step 1 (value + 1 = the sum so far), and the fused layer kernel's launch
// counter.
enum : int {
  kCtlItems = 1,
  kCtlBar = 2,
  kCtlAbort = 5,
  kCtlTot = 8,
  kCtlLaunches = kCtlTot + kAgg + 1,  // 64-bit launch counter of the fused layer kernel (8-byte aligned)
  kCtlWords = kCtlLaunches + 2
};

// The grouping of one batch (the caller's buffer, carved by carve_ws).
struct GroupWs {
  int* key;       // [hcap] id in the slot, -1 = empty
  int* cnt;       // [hcap] tokens in the slot minus one
  unsigned* ctl;  // [kCtlWords]
  int* off;       // [hcap] first list position of the slot's tokens
  int* tok_slot;  // [T] slot of token t (-1 for a bad id)
  int* tok_rank;  // [T] rank of token t in its id's group
  int* tok_pos;   // [T] list position of token t (-1 for a bad id)
  int* list;      // [T] tokens grouped by id
  int4* items;    // [T + T / kItemTokens + 1] {id, first list position, tokens, dense index of the id}
  int* uid_id;    // [T] the id of each dense index (distinct ids numbered 0..U-1)
  int* slot_uid;  // [hcap] dense index of the slot's id
  int* tok_uid;   // [T] dense index of token t's id (-1 for a bad id)
  float* gates;   // [T][NP] one layer's gates by list position
  unsigned* tile_flag;  // [ceil(T / 16)] the fused layer kernel's router-tile flags
  int hcap_log2;
  size_t clear_bytes;  // key .. ctl .. tile_flag, one contiguous range
};

int padded_experts(int N) { return N <= 8 ? 8 : N <= 16 ? 16 : 32; }

// Carves the buffer at `base` (nullptr: size query); returns its size.
size_t carve_ws(void* base, int64_t T, int NP, GroupWs* w) {
  int lg = 10;
  while ((int64_t(1) << lg) < 2 * T) ++lg;
  const int64_t hcap = int64_t(1) << lg;
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  const size_t n_flags = (size_t)((T + 15) / 16);
  const size_t clear = 8 * (size_t)hcap + 4 * kCtlWords + 4 * n_flags;
  const size_t o_clear = take(clear);
  const size_t o_off = take(4 * (size_t)hcap);
  const size_t o_tslot = take(4 * (size_t)T);
  const size_t o_trank = take(4 * (size_t)T);
  const size_t o_tpos = take(4 * (size_t)T);
  const size_t o_list = take(4 * (size_t)T);
  const size_t o_items = take(16 * (size_t)(T + T / kItemTokens + 1));
  const size_t o_uid = take(4 * (size_t)T);
  const size_t o_suid = take(4 * (size_t)hcap);
  const size_t o_tuid = take(4 * (size_t)T);
  const size_t o_gates = take(4 * (size_t)T * NP);
  if (w != nullptr && base != nullptr) {
    uint8_t* b = static_cast<uint8_t*>(base);
    w->key = reinterpret_cast<int*>(b + o_clear);
    w->cnt = w->key + hcap;
    w->ctl = reinterpret_cast<unsigned*>(w->cnt + hcap);
    w->tile_flag = w->ctl + kCtlWords;
    w->off = reinterpret_cast<int*>(b + o_off);
    w->tok_slot = reinterpret_cast<int*>(b + o_tslot);
    w->tok_rank = reinterpret_cast<int*>(b + o_trank);
    w->tok_pos = reinterpret_cast<int*>(b + o_tpos);
    w->list = reinterpret_cast<int*>(b + o_list);
    w->items = reinterpret_cast<int4*>(b + o_items);
    w->uid_id = reinterpret_cast<int*>(b + o_uid);
    w->slot_uid = reinterpret_cast<int*>(b + o_suid);
    w->tok_uid = reinterpret_cast<int*>(b + o_tuid);
    w->gates = reinterpret_cast<float*>(b + o_gates);
    w->hcap_log2 = lg;
    w->clear_bytes = clear;
  }
  return off;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}


}  // namespace
}  // namespace mole
