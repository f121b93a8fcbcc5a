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
// the three grid-barrier counters, the abort word, the CTA count the shares
// were built for, and the running totals of step 1 (value + 1 = the sum so
// far).
enum : int {
  kCtlItems = 1,
  kCtlBar = 2,
  kCtlAbort = 5,
  kCtlShareGrid = 6,
  kCtlTot = 8,
  kCtlWords = kCtlTot + kAgg + 1
};

// Shares: the work items of each CTA of a one-CTA-per-SM layer kernel (G
// CTAs, G <= kShareGridMax), in that CTA's processing order, with their
// tokens.  A CTA's items number at most, and its tokens at most, share_cap
// (items are laid out largest first and dealt in rounds of G: the CTA's item
// of round m >= 1 is no larger than any item of round m-1, so its tokens
// number at most kItemTokens + T / G); shares are built when that is below
// kShareCapLimit.
constexpr int kShareGridMax = 256;
constexpr int kShareCapLimit = 256;

__host__ __device__ constexpr int64_t share_cap(int64_t T, int64_t G) {
  return (kItemTokens + (T + G - 1) / G + 15) / 16 * 16;
}

// Bound on G * share_cap(T, G) over G <= kShareGridMax.
__host__ __device__ constexpr int64_t share_words(int64_t T) { return T + 33 * (int64_t)kShareGridMax; }

__host__ __device__ constexpr bool shares_apply(int64_t T, int64_t G) {
  return G >= 1 && G <= kShareGridMax && share_cap(T, G) < kShareCapLimit;
}

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
  int* share_n;     // [kShareGridMax][2] per layer CTA b: work items, tokens
  int4* share_rec;  // item records of CTA b at b * cap, in its processing order (cap = share_cap(T, G))
  int* share_tok;   // tokens of those items, in order, CTA b's at b * cap
  int* share_off;   // CTA b's token offset of each step (and the total) at b * (cap + 1)
  int hcap_log2;
  size_t clear_bytes;  // key .. ctl, one contiguous range
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
  const size_t clear = 8 * (size_t)hcap + 4 * kCtlWords;
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
  const size_t o_sn = take(8 * (size_t)kShareGridMax);
  const size_t o_srec = take(16 * (size_t)share_words(T));
  const size_t o_stok = take(4 * (size_t)share_words(T));
  const size_t o_soff = take(4 * ((size_t)share_words(T) + kShareGridMax));
  // last: the only region whose size depends on NP (a grouping serves
  // layers with any expert count up to the one it was sized for)
  const size_t o_gates = take(4 * (size_t)T * NP);
  if (w != nullptr && base != nullptr) {
    uint8_t* b = static_cast<uint8_t*>(base);
    w->key = reinterpret_cast<int*>(b + o_clear);
    w->cnt = w->key + hcap;
    w->ctl = reinterpret_cast<unsigned*>(w->cnt + hcap);
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
    w->share_n = reinterpret_cast<int*>(b + o_sn);
    w->share_rec = reinterpret_cast<int4*>(b + o_srec);
    w->share_tok = reinterpret_cast<int*>(b + o_stok);
    w->share_off = reinterpret_cast<int*>(b + o_soff);
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
