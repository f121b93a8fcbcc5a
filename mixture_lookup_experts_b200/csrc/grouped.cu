// grouped.cu -- lookup-combine with the batch's tokens grouped by token id
// (MoLE page, 推理阶段 and 复杂度分析: what moves per token is its block of N
// expert-output rows, addressed by the token id).  A prefill batch of text
// repeats ids -- with Zipf-distributed ids, 16384 tokens over a 50K
// vocabulary hold about 4K distinct ids -- and every token with the same id
// reads the same row block.  This path fetches each distinct row block once
// per batch and combines all of that id's tokens from one shared-memory copy.
// Every MoLE layer indexes its table with the same input token ids, so the
// grouping is built once per batch and serves all layers.
//
//  1. group_plan_kernel (cooperative launch; once per batch):
//       step 0  every token's id goes into an open-addressing hash table
//               (one atomicCAS per distinct id of a warp), and the token
//               takes a rank inside its id's group (one atomicAdd per
//               distinct slot of a warp, __match_any_sync);
//       step 1  per CTA, the token and work-item totals (by item size) of a
//               range of table slots (an item = up to kItemTokens tokens of
//               one id), added atomically to grid totals: the running total
//               a CTA sees is its base inside each region;
//       step 2  per id the offset of its token range in the list and its
//               item records, laid out by item size, largest first;
//       step 3  every token's list position: list[pos] = t, tok_pos[t] = pos.
//     Steps 1-3 each start after a grid-wide barrier (bounded wait).
//     Then group_share_kernel (once per batch) lists, for each CTA of a
//     one-CTA-per-SM layer kernel, its work items in processing order and
//     their tokens (its share).
//  Per layer, bf16 table, batches of at least about 3/4 of a 128-token tile
//  per SM (the prefill sizes):
//  2. grouped_stream_kernel (one CTA per SM, 9 warps): the CTA's share
//     streams through one ring of shared-memory slots as two kinds of
//     entries -- a router tile (16 of its tokens' h rows) placed just ahead
//     of the first work item that needs it, and each work item's row block --
//     so h and the row blocks come from memory together; the consumer warps
//     turn a tile into gates (mma.sync router, gates kept in shared memory)
//     and combine an item as in 3.
//  Per layer, smaller batches (bf16 or NF3 table):
//  2. grouped_local_kernel (one CTA per SM, 9 warps): each CTA computes the
//     gates of its own share's tokens first, then gathers and combines its
//     work items as in 3.
//  Per layer, NF3 table at the prefill sizes (or where neither applies):
//  2. the router: router_tc.cu's tcgen05 kernel for an NF3 table with 16
//     experts, else router_group_kernel (persistent, 2 CTAs per SM, the
//     mma.sync router of combine_common.cuh); each token's gates go to its
//     list position, so an item's gates are contiguous.
//  3. grouped_gather_kernel (one CTA per SM, 9 warps): a producer warp
//     copies each work item's row block and its tokens' gates (two
//     cp.async.bulk) into a ring of shared-memory slots; 8 consumer warps
//     convert each 4-element vector of the N rows to fp32 once and apply it
//     to every token of the item.
//
// Per token the arithmetic is that of the ungrouped kernels (the same router
// code, then out = sum over j = 0..N-1, in order, of g_j * x_j with fp32
// FMAs), so both paths give bit-identical outputs; only the order in which
// tokens are processed differs.
#include "groups.cuh"

namespace mole {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanMaxGrid = 1024;
constexpr int64_t kGroupedMinT = 1024;
constexpr int64_t kGroupedMaxT = kMaxOffloadT;

// Grid-wide barrier of a cooperative launch, split in two so that work can
// run between the arrival and the wait; `counter` starts at 0xFFFFFFFF and
// serves one barrier per call.  grid_arrive publishes this CTA's earlier
// writes and counts it in.
__device__ __forceinline__ void grid_arrive(unsigned* counter) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) atomicAdd(counter, 1u);
}

// Waits until every CTA has arrived.  Bounded: after kWaitLimitNs, or when
// another CTA has given up, it returns false (the giving-up CTA sets the
// abort word and the timeout bit).
__device__ bool grid_wait(unsigned* counter, unsigned* abort_word, unsigned* err, int* flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned target = gridDim.x - 1u;
    if (ld_acquire(counter) != target) {
      const uint64_t t0 = globaltimer();
      while (ld_acquire(counter) != target) {
        if (ld_acquire(abort_word) != 0xFFFFFFFFu) {
          ok = 0;
          break;
        }
        if (globaltimer() - t0 > kWaitLimitNs) {
          atomicExch(abort_word, 1u);
          atomicOr(err, kErrTimeout);
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    *flag = ok;
  }
  __syncthreads();
  return *flag != 0;
}

// Exclusive scan of (a, b) over the CTA in thread order; totals in (ta, tb).
// `red` holds 2 * kWarps ints.
__device__ __forceinline__ void block_scan2(int& a, int& b, int& ta, int& tb, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, ia, o), y = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += x;
      ib += y;
    }
  }
  if (lane == 31) {
    red[2 * warp] = ia;
    red[2 * warp + 1] = ib;
  }
  __syncthreads();
  int wa = 0, wb = 0, sa = 0, sb = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int x = red[2 * w], y = red[2 * w + 1];
    if (w < warp) {
      wa += x;
      wb += y;
    }
    sa += x;
    sb += y;
  }
  __syncthreads();
  a = wa + ia - a;
  b = wb + ib - b;
  ta = sa;
  tb = sb;
}

// Slot of `id` in the hash table (linear probing), inserting it if new.
__device__ __forceinline__ int plan_insert(const GroupWs& w, int id) {
  const unsigned mask = (1u << w.hcap_log2) - 1u;
  unsigned hh = ((unsigned)id * 2654435761u) >> (32 - w.hcap_log2);
  for (unsigned probe = 0; probe <= mask; ++probe) {
    const int k = atomicCAS(&w.key[hh], -1, id);
    if (k == -1 || k == id) return (int)hh;
    hh = (hh + 1u) & mask;
  }
  return -1;  // not reached: the table has at least 2T slots
}

// This CTA's range [s0, s1) of hash-table slots.
__device__ __forceinline__ void slot_range(const GroupWs& w, int64_t& s0, int64_t& s1) {
  const int64_t hcap = int64_t(1) << w.hcap_log2;
  s0 = (int64_t)blockIdx.x * hcap / gridDim.x;
  s1 = ((int64_t)blockIdx.x + 1) * hcap / gridDim.x;
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Step 1: token, per-size item and distinct-id totals of this CTA's slot
// range, added to the grid totals; the values the totals had before (in
// whatever order the CTAs arrive) become this CTA's bases within each region.
// `cls` and `cbase` are kAgg + 1 ints of shared memory.
__device__ void plan_count(const GroupWs& w, int* cls, int* cbase) {
  int64_t s0, s1;
  slot_range(w, s0, s1);
  if (threadIdx.x <= kAgg) cls[threadIdx.x] = 0;
  __syncthreads();
  int sc = 0, su = 0;
  for (int64_t h = s0 + threadIdx.x; h < s1; h += kThreads) {
    if (w.key[h] == -1) continue;
    const int c = w.cnt[h] + 1;
    sc += c;
    ++su;
    if (c >= kItemTokens) atomicAdd(&cls[kItemTokens], c / kItemTokens);
    if (c % kItemTokens) atomicAdd(&cls[c % kItemTokens], 1);
  }
  sc = warp_sum(sc);
  su = warp_sum(su);
  if ((threadIdx.x & 31) == 0 && sc) atomicAdd(&cls[0], sc);
  if ((threadIdx.x & 31) == 0 && su) atomicAdd(&cls[kAgg], su);
  __syncthreads();
  if (threadIdx.x <= kAgg) {
    const int v = cls[threadIdx.x];
    cbase[threadIdx.x] = v ? (int)(atomicAdd(&w.ctl[kCtlTot + threadIdx.x], (unsigned)v) + 1u) : 0;
  }
}

// Step 2: list offsets and item records of this CTA's slot range.  Items are
// laid out by size, largest first (all full items, then 15-token items, ...),
// so dealing them to the gather CTAs in alternating rounds spreads the tokens evenly.
// `cur` is kAgg ints of shared memory, `red` 2 * kWarps.
__device__ void plan_offsets(const GroupWs& w, const int* cbase, int* cur, int* red) {
  int64_t s0, s1;
  slot_range(w, s0, s1);
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int n = kItemTokens; n >= 1; --n) {
      cur[n] = acc + cbase[n];
      acc += (int)(ld_relaxed_u32(&w.ctl[kCtlTot + n]) + 1u);  // ordered by the grid barrier
    }
    if (blockIdx.x == 0) w.ctl[kCtlItems] = (unsigned)acc;
  }
  __syncthreads();
  int bt = cbase[0], bu = cbase[kAgg];
  for (int64_t base = s0; base < s1; base += kThreads) {
    const int64_t h = base + threadIdx.x;
    const int id = h < s1 ? w.key[h] : -1;
    const int c = id != -1 ? w.cnt[h] + 1 : 0;
    int pc = c, pu = id != -1 ? 1 : 0, sc, su;
    block_scan2(pc, pu, sc, su, red);
    if (id != -1) {
      const int o = bt + pc, uid = bu + pu;
      w.off[h] = o;
      w.slot_uid[h] = uid;
      w.uid_id[uid] = id;
      const int nf = c / kItemTokens, r = c % kItemTokens;
      if (nf) {
        const int p0 = atomicAdd(&cur[kItemTokens], nf);
        for (int k = 0; k < nf; ++k) w.items[p0 + k] = make_int4(id, o + k * kItemTokens, kItemTokens, uid);
      }
      if (r) w.items[atomicAdd(&cur[r], 1)] = make_int4(id, o + nf * kItemTokens, r, uid);
    }
    bt += sc;
    bu += su;
  }
}

// This CTA's contiguous range [t0, t1) of the batch's tokens.
__device__ __forceinline__ void token_range(int64_t T, int64_t& t0, int64_t& t1) {
  t0 = (int64_t)blockIdx.x * T / gridDim.x;
  t1 = ((int64_t)blockIdx.x + 1) * T / gridDim.x;
}

// Step 0: insert this CTA's tokens and rank them inside their id's group.
__device__ void plan_insert_tokens(const int32_t* __restrict__ ids, int64_t T, int64_t V, const GroupWs& w,
                                   unsigned* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t t0, t1;
  token_range(T, t0, t1);
  for (int64_t base = t0 + (int64_t)warp * 32; base < t1; base += kPlanThreads) {
    const int64_t t = base + lane;
    const bool act = t < t1;
    const int id = act ? __ldg(ids + t) : -1;
    const bool good = act && id >= 0 && (int64_t)id < V;
    if (act && !good) atomicOr(err, kErrIndex);
    // one insert per distinct id of the warp (the leader's), shared by shuffle
    const unsigned same = __match_any_sync(0xffffffffu, good ? id : -1);
    const int lead = __ffs(same) - 1;
    int slot = (good && lane == lead) ? plan_insert(w, id) : -1;
    slot = __shfl_sync(0xffffffffu, slot, lead);
    if (!good) slot = -1;
    // one atomicAdd per distinct slot of the warp; ranks by lane order
    const unsigned peers = __match_any_sync(0xffffffffu, slot);
    const int leader = __ffs(peers) - 1;
    int first = 0;
    if (slot >= 0 && lane == leader) first = atomicAdd(&w.cnt[slot], __popc(peers)) + 1;
    first = __shfl_sync(0xffffffffu, first, leader);
    if (act) {
      w.tok_slot[t] = slot;
      w.tok_rank[t] = first + __popc(peers & ((1u << lane) - 1u));
    }
  }
}

// Step 3: every token of this CTA to its list position (and its id's dense
// index).
__device__ void plan_scatter(const GroupWs& w, int64_t T) {
  int64_t t0, t1;
  token_range(T, t0, t1);
  for (int64_t t = t0 + threadIdx.x; t < t1; t += kPlanThreads) {
    const int slot = w.tok_slot[t];
    const int pos = slot >= 0 ? w.off[slot] + w.tok_rank[t] : -1;
    w.tok_pos[t] = pos;
    w.tok_uid[t] = slot >= 0 ? w.slot_uid[slot] : -1;
    if (pos >= 0) w.list[pos] = (int)t;
  }
}

__global__ void __launch_bounds__(kPlanThreads) group_plan_kernel(const int32_t* __restrict__ ids, int64_t T,
                                                                   int64_t V, const GroupWs w, unsigned* err) {
  __shared__ int red[2 * kWarps];
  __shared__ int cls[kAgg + 1], cbase[kAgg + 1];
  __shared__ int flag;
  plan_insert_tokens(ids, T, V, w, err);
  grid_arrive(&w.ctl[kCtlBar + 0]);
  bool ok = grid_wait(&w.ctl[kCtlBar + 0], &w.ctl[kCtlAbort], err, &flag);
  if (ok) plan_count(w, cls, cbase);
  grid_arrive(&w.ctl[kCtlBar + 1]);
  if (ok) ok = grid_wait(&w.ctl[kCtlBar + 1], &w.ctl[kCtlAbort], err, &flag);
  if (ok) plan_offsets(w, cbase, cls, red);
  grid_arrive(&w.ctl[kCtlBar + 2]);
  if (ok) ok = grid_wait(&w.ctl[kCtlBar + 2], &w.ctl[kCtlAbort], err, &flag);
  if (ok) plan_scatter(w, T);
}

struct GArgs {
  int64_t T;
  const uint16_t* h;
  const uint16_t* Wr;
  const uint16_t* table;    // bf16 table
  const uint8_t* codes;     // NF3 table: codes and fp16 scales
  const uint16_t* scales;
  int N, D;
  float* out;
  unsigned* err;
  // by_uid: the table holds the batch's distinct ids' row blocks by dense
  // index (a staging buffer of `rows` blocks), not the whole vocabulary
  int by_uid;
  int64_t rows;
};

// One layer's router: gates to the tokens' list positions; a token with a
// bad id gets a NaN output row (and the index bit of the error word).
template <int NT>
__global__ void __launch_bounds__(kThreads, 2) router_group_kernel(const GArgs p, const GroupWs w) {
  constexpr int NP = 8 * NT;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Smem s = carve<true, NP>(smem_raw, p.D);
  // list positions of the tile's tokens, loaded one tile ahead (thread r <
  // 16); the first tile's inside the first sink, after router_tiles has
  // waited for the previous kernel (it may be the one building the grouping)
  int pos_next = -1;
  bool first = true;
  router_tiles<NT>(s, p.h, p.Wr, p.T, p.N, p.D, [&](int64_t t0, int rows) {
    if (threadIdx.x < kTileMax) {
      if (first && t0 + threadIdx.x < p.T) pos_next = w.tok_pos[t0 + threadIdx.x];
      s.tok_id[threadIdx.x] = pos_next;
      const int64_t tn = t0 + (int64_t)gridDim.x * kTileMax + threadIdx.x;
      pos_next = tn < p.T ? w.tok_pos[tn] : -1;
    }
    first = false;
    __syncthreads();
    for (int i = threadIdx.x; i < rows * NP; i += kThreads) {
      const int r = i / NP, j = i - r * NP;
      const int pos = s.tok_id[r];
      if (pos >= 0) w.gates[(int64_t)pos * NP + j] = s.gates[i];
    }
    for (int r = 0; r < rows; ++r) {
      if (s.tok_id[r] >= 0) continue;
      if (threadIdx.x == 0) atomicOr(p.err, kErrIndex);
      float* o = p.out + (t0 + r) * p.D;
      for (int d = 4 * threadIdx.x; d < p.D; d += 4 * kThreads)
        __stcs(reinterpret_cast<float4*>(o + d), make_float4(NAN, NAN, NAN, NAN));
    }
  });
}

// Slot layout: [0, gates_off) the id's row block (N rows of D bf16),
// [gates_off, + kItemTokens * NP * 4) the gates of the item's tokens.
struct GroupLayout {
  int n_slots, slot_bytes, gates_off, scales_off;  // scales_off: NF3 table only
};

// 8 consumer warps + 1 producer warp: 3 warps per scheduler, so a thread may
// hold 168 registers -- the N rows of its 4-element vector stay in registers
// in fp32 (up to 16 experts) while it serves every token of the item.
constexpr int kGroupCons = 8;

// bf16 -> fp32 through opaque instructions: the compiler keeps the converted
// values in registers across the item's tokens instead of converting again
// per token (which it otherwise prefers, to save registers).
__device__ __forceinline__ float bf16_lo_held(uint32_t x) {
  uint32_t u;
  asm volatile("shl.b32 %0, %1, 16;" : "=r"(u) : "r"(x));
  return __uint_as_float(u);
}
__device__ __forceinline__ float bf16_hi_held(uint32_t x) {
  uint32_t u;
  asm volatile("and.b32 %0, %1, 0xffff0000;" : "=r"(u) : "r"(x));
  return __uint_as_float(u);
}
constexpr int kGroupThreads = (kGroupCons + 1) * 32;
constexpr int kGroupProducer = kGroupCons;

// Packed fp32 FMA (two lanes per instruction, each rounded as fmaf): the
// gate g times an element pair, plus the pair's running sums.
__device__ __forceinline__ float2 ffma2(float g, float2 x, float2 acc) {
  return __ffma2_rn(make_float2(g, g), x, acc);
}

// out[t, 4v .. 4v+3] for one token from the N rows of the unit (x, fp32
// pairs or packed bf16 pairs) and the token's gates g (NP floats in shared
// memory).  Per element the FMAs run over j = 0..N-1 in order.
template <int NP, bool kExactN, bool kPacked>
__device__ __forceinline__ float4 combine_unit(const float2 (&xf)[kPacked ? 1 : NP][2], const uint2 (&xp)[kPacked ? NP : 1],
                                               const float* g, int N) {
  const float4* g4 = reinterpret_cast<const float4*>(g);
  float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
  for (int jq = 0; jq < NP / 4; ++jq) {
    const float4 gv = g4[jq];
    const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * jq + e;
      if (kExactN || j < N) {
        if (kPacked) {
          const uint2 r = xp[kPacked ? j : 0];
          a01 = ffma2(gg[e], make_float2(bf16_lo(r.x), bf16_hi(r.x)), a01);
          a23 = ffma2(gg[e], make_float2(bf16_lo(r.y), bf16_hi(r.y)), a23);
        } else {
          a01 = ffma2(gg[e], xf[kPacked ? 0 : j][0], a01);
          a23 = ffma2(gg[e], xf[kPacked ? 0 : j][1], a23);
        }
      }
    }
  }
  return make_float4(a01.x, a01.y, a23.x, a23.y);
}

// out for 4 tokens at once (gates at g + k * gstride floats, k = 0..3):
// 16 independent FMA chains (8 packed pairs) over the N rows held in fp32.
template <int NP, bool kExactN>
__device__ __forceinline__ void combine_quad(const float2 (&xf)[NP][2], const float* g, int gstride, int N,
                                             float2 (&o)[4][2]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) o[k][0] = o[k][1] = make_float2(0.f, 0.f);
#pragma unroll
  for (int jq = 0; jq < NP / 4; ++jq) {
    float4 gv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) gv[k] = reinterpret_cast<const float4*>(g + k * gstride)[jq];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * jq + e;
      if (kExactN || j < N) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float gk = e == 0 ? gv[k].x : e == 1 ? gv[k].y : e == 2 ? gv[k].z : gv[k].w;
          o[k][0] = ffma2(gk, xf[j][0], o[k][0]);
          o[k][1] = ffma2(gk, xf[j][1], o[k][1]);
        }
      }
    }
  }
}

// The NF3 table's counterparts: row j's 4 elements hold the levels, sc[j] the
// block scale; per token the gate and the scale are multiplied first and the
// product scales the levels, as the ungrouped kernels do.
template <int NP, bool kExactN>
__device__ __forceinline__ void combine_quad_nf3(const float2 (&xf)[NP][2], const float (&sc)[NP], const float* g,
                                                 int gstride, int N, float2 (&o)[4][2]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) o[k][0] = o[k][1] = make_float2(0.f, 0.f);
#pragma unroll
  for (int jq = 0; jq < NP / 4; ++jq) {
    float4 gv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) gv[k] = reinterpret_cast<const float4*>(g + k * gstride)[jq];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * jq + e;
      if (kExactN || j < N) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = (e == 0 ? gv[k].x : e == 1 ? gv[k].y : e == 2 ? gv[k].z : gv[k].w) * sc[j];
          o[k][0] = ffma2(a, xf[j][0], o[k][0]);
          o[k][1] = ffma2(a, xf[j][1], o[k][1]);
        }
      }
    }
  }
}

template <int NP, bool kExactN>
__device__ __forceinline__ float4 combine_unit_nf3(const float2 (&xf)[NP][2], const float (&sc)[NP], const float* g,
                                                   int N) {
  float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    if (kExactN || j < N) {
      const float a = g[j] * sc[j];
      a01 = ffma2(a, xf[j][0], a01);
      a23 = ffma2(a, xf[j][1], a23);
    }
  }
  return make_float4(a01.x, a01.y, a23.x, a23.y);
}

__device__ __forceinline__ float held(float x) {
  uint32_t u;
  asm volatile("mov.b32 %0, %1;" : "=r"(u) : "r"(__float_as_uint(x)));
  return __uint_as_float(u);
}

// Levels of the 4 NF3 codes in the low 12 bits of x.
__device__ __forceinline__ void nf3_levels4(uint32_t x, float (&f)[4]) {
  uint32_t sl, sh;
  nf3_selectors(x, sl, sh);
  const uint32_t lo = prmt(kLoBytes0, kLoBytes1, sl);
  const uint32_t hi = prmt(kHiBytes0, kHiBytes1, sl);
  const uint32_t h01 = prmt(lo, hi, 0x5140u);
  const uint32_t h23 = prmt(lo, hi, 0x7362u);
  const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  f[0] = f01.x;
  f[1] = f01.y;
  f[2] = f23.x;
  f[3] = f23.y;
}

// The ring of work items in shared memory: n_slots slots of slot_bytes, then
// per slot a `full` barrier (three arrivals: the row block's copies, the
// gates' copy, the token list -- each copy arrival with its byte count), an
// `empty` barrier (one arrival per consumer warp), the item's token count and
// token list; then the CTA's abort flag.
struct Ring {
  uint8_t* slots;
  uint64_t* full;
  uint64_t* empty;
  int* slot_n;
  int* slot_tok;  // [n_slots][kItemTokens]
  int* abort;
};

__host__ __device__ constexpr size_t ring_bytes(int n_slots, int slot_bytes) {
  return (size_t)n_slots * slot_bytes + (size_t)n_slots * (16 + 4 + 4 * kItemTokens) + 16;
}

__device__ __forceinline__ Ring carve_ring(uint8_t* base, const GroupLayout& L) {
  Ring r;
  r.slots = base;
  r.full = reinterpret_cast<uint64_t*>(base + (size_t)L.n_slots * L.slot_bytes);
  r.empty = r.full + L.n_slots;
  r.slot_n = reinterpret_cast<int*>(r.empty + L.n_slots);
  r.slot_tok = r.slot_n + L.n_slots;
  r.abort = r.slot_tok + L.n_slots * kItemTokens;
  return r;
}

// Thread 0: barriers initialised (`full_arrivals` per full phase), abort
// flag cleared.
__device__ __forceinline__ void ring_init(const Ring& r, const GroupLayout& L, int full_arrivals = 3) {
  for (int q = 0; q < L.n_slots; ++q) {
    mbar_init(&r.full[q], full_arrivals);
    mbar_init(&r.empty[q], kGroupCons);
  }
  *r.abort = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// The CTA-local layer kernel's router inputs.  Wr arrives by bulk copies in
// the ring's last slots wr_slot0 .. n_slots-1 (one slot of a bf16 table; the
// smaller slots of an NF3 table take several) (wr_full) and goes back to the
// ring once every consumer warp holds its B fragments in registers
// (wr_free).  Where the slots before them can hold a 16-token tile of h rows
// (pitch bytes apart), the router tiles stream through those staging slots
// st_slot0 .. wr_slot0-1 one at a time, one bulk copy per row (h_full, one
// phase per tile), each released once its MMAs are done (h_empty); after
// the last tile they go back to the ring.  The CTA's work item records and
// tokens come from its share, in processing order.
struct LocalSync {
  uint64_t* wr_full;
  uint64_t* wr_free;
  uint64_t* h_full;
  uint64_t* h_empty;
  const int4* recs;  // [my_n]
  const int* tok;    // [n_tok]
  int wr_slot0;
  int st_slot0;      // == wr_slot0: no staging slots (A fragments from global memory)
  int n_st;          // router tiles staged (all of them, or none)
  int n_tok;
  int pitch;
};

// Ring slots that hold Wr in the CTA-local kernel: the last ones, as many as
// its N * D bf16 values need.
__host__ __device__ __forceinline__ int wr_slots(const GroupLayout& L, int N, int D) {
  return (int)(((int64_t)N * D * 2 + L.slot_bytes - 1) / L.slot_bytes);
}

// Ring position of the CTA's k-th work item: slot k mod n_slots, in lap
// k / n_slots.
__device__ __forceinline__ uint32_t ring_slot(const Ring&, const GroupLayout& L, int k) {
  return (uint32_t)(k % L.n_slots);
}
__device__ __forceinline__ uint32_t ring_parity(const GroupLayout& L, int k) {
  return (uint32_t)((k / L.n_slots) & 1);
}

// The work items (largest first) are dealt to the G CTAs of a layer kernel in
// rounds of G, alternating direction (round m: CTA b takes the item at
// position b of the round if m is even, G - 1 - b if odd), so that no CTA
// takes the largest item of every round.
__host__ __device__ __forceinline__ int item_of(int m, int b, int G) { return m * G + ((m & 1) ? G - 1 - b : b); }

__host__ __device__ __forceinline__ int items_of(int n_items, int b, int G) {
  const int full = n_items / G;  // complete rounds
  return full + (item_of(full, b, G) < n_items ? 1 : 0);
}

// CTA b's work item at step k of its processing order: those of rounds 0,
// my_n-1, 1, my_n-2, ... (large, small, large, ...).
__host__ __device__ __forceinline__ int cta_item(int k, int my_n, int b, int G) {
  return item_of((k & 1) ? my_n - 1 - (k >> 1) : (k >> 1), b, G);
}

__device__ __forceinline__ int items_of_cta(const GroupWs& w) {
  return items_of((int)ld_relaxed_u32(&w.ctl[kCtlItems]), (int)blockIdx.x, (int)gridDim.x);
}

// Producer warp of the gather.  The CTA's work items are taken in cta_item
// order, so the copies of small items proceed while the consumers work
// through large ones.  Item records are read 32 at a time (one per lane) and
// each item's token list one item ahead.  Per item: the row block's copies
// and (grouped_gather_kernel) its tokens' gates into the item's slot, then
// the token list.  With `ls` (CTA-local kernel, gates in shared memory) the
// records come from the CTA's share, the row blocks of the first items go
// out at once (those of Wr's slots once Wr is no longer needed there), and
// the warp
// also writes the
// NaN output rows of the bad-id tokens in its CTA's slice of the batch.
template <int NP, bool kNf3>
__device__ void ring_producer(const GArgs& p, const GroupWs& w, const GroupLayout& L, const Ring& r, int my_n,
                              const LocalSync* ls, int tok0 = 0) {
  constexpr int C = kItemTokens;
  const int lane = threadIdx.x & 31;
  volatile int* abort = r.abort;
  const uint32_t row_bytes = (uint32_t)p.N * (uint32_t)p.D * 2u;
  const int NB = p.D >> 6;  // NF3 blocks per row
  const uint32_t code_bytes = (uint32_t)p.N * (uint32_t)NB * 24u, scale_bytes = (uint32_t)p.N * (uint32_t)NB * 2u;
  auto record = [&](int kk) {
    if (kk >= my_n) return make_int4(0, 0, 0, 0);
    return ls != nullptr ? ls->recs[kk] : w.items[cta_item(kk, my_n, (int)blockIdx.x, (int)gridDim.x)];
  };
  // the row block's copies into slot q, on its full barrier (lane 0)
  auto issue_rows = [&](uint32_t q, int row) {
    uint8_t* slot = r.slots + (size_t)q * L.slot_bytes;
    if (lane == 0) {
      if (kNf3) {
        mbar_expect_tx(&r.full[q], code_bytes + scale_bytes);
        bulk_g2s(slot, p.codes + (int64_t)row * code_bytes, code_bytes, &r.full[q]);
        bulk_g2s(slot + L.scales_off, p.scales + (int64_t)row * p.N * NB, scale_bytes, &r.full[q]);
      } else {
        mbar_expect_tx(&r.full[q], row_bytes);
        bulk_g2s(slot, p.table + (int64_t)row * p.N * p.D, row_bytes, &r.full[q]);
      }
    }
  };
  auto bad_row = [&](int row) {  // staging buffer smaller than the batch's distinct ids
    if (!p.by_uid || (int64_t)row < p.rows) return false;
    if (lane == 0) atomicOr(p.err, kErrIndex);
    *abort = 1;
    return true;
  };
  // items 0 .. issued-1 went out in full
  int issued = 0;
  // records of steps k0 + lane (my_item) and k0 + 32 + lane (nx_item)
  int k0 = 0;
  int4 my_item = record(lane);
  int4 nx_item = record(32 + lane);
  bool ok = true;
  int pre = 0;  // items whose row blocks went out ahead of the main loop
  int staged = 0;  // router tiles whose h rows went out
  if (ls != nullptr) {
    // router tile t's h rows into the staging slots, lane r copying row r
    // (its token id tk)
    uint8_t* stage = r.slots + (size_t)ls->st_slot0 * L.slot_bytes;
    const uint32_t h_row = (uint32_t)p.D * 2u;
    auto stage_tile = [&](int t, int tk) {
      const int rows = ls->n_tok - t * kTileMax < kTileMax ? ls->n_tok - t * kTileMax : kTileMax;
      if (lane == 0) mbar_expect_tx(ls->h_full, (uint32_t)rows * h_row);
      __syncwarp();
      if (lane < rows) bulk_g2s(stage + (size_t)lane * ls->pitch, p.h + (int64_t)tk * p.D, h_row, ls->h_full);
    };
    // the remaining tiles, each once the previous one's MMAs are done
    auto stage_rest = [&]() {
      for (; staged < ls->n_st; ++staged) {
        const int i = staged * kTileMax + lane;
        const int tk = lane < kTileMax && i < ls->n_tok ? __ldg(ls->tok + i) : 0;
        if (!warp_wait(ls->h_empty, (uint32_t)((staged - 1) & 1), abort, p.err)) return false;
        stage_tile(staged, tk);
      }
      return true;
    };
    if (ls->n_st > 0) {
      stage_tile(0, tok0);
      staged = 1;
    }
    // the first lap (item k in slot k): the free slots at once, then Wr's
    // slots once the B fragments are in registers, then the staging slots
    // after the router's last tile
    const int first = my_n < L.n_slots ? my_n : L.n_slots;  // n_slots <= 16 < 32: all in my_item
    uint32_t sent = 0;  // lap-0 items whose row blocks went out
    for (int pass = 0; ok && pass < 3; ++pass) {
      for (int k = 0; k < first; ++k) {
        const int q = (int)ring_slot(r, L, k);
        const int kind = q >= ls->wr_slot0 ? 1 : (q >= ls->st_slot0 && ls->n_st > 0 ? 2 : 0);
        if (kind != pass) continue;
        const int row = __shfl_sync(0xffffffffu, p.by_uid ? my_item.w : my_item.x, k);
        if (bad_row(row)) {
          ok = false;
          break;
        }
        if (kind == 1)
          ok = warp_wait(ls->wr_free, 0u, abort, p.err);
        else if (kind == 2)
          ok = stage_rest() && warp_wait(ls->h_empty, (uint32_t)((ls->n_st - 1) & 1), abort, p.err);
        if (!ok) break;
        issue_rows((uint32_t)q, row);
        sent |= 1u << k;
      }
    }
    if (ok) ok = stage_rest();  // (fewer items than slots)
    pre = first;
    if (!ok) {
      // the lap-0 items sent hold row copies but no token list: their
      // missing arrivals, so their phases complete when the copies land,
      // then wait for those (the consumers see the abort flag)
      *abort = 1;
      __syncwarp();
      if (lane == 0) {
        for (int kk = 0; kk < first; ++kk)
          if (sent >> kk & 1u) mbar_arrive(&r.full[ring_slot(r, L, kk)]);
        for (int kk = 0; kk < first; ++kk)
          if (sent >> kk & 1u) mbar_drain(&r.full[ring_slot(r, L, kk)], 0u);
      }
      issued = 0;
    }
  }
  int next_tok = -1;
  if (my_n > 0 && ok) {
    const int pos = __shfl_sync(0xffffffffu, my_item.y, 0), n = __shfl_sync(0xffffffffu, my_item.z, 0);
    next_tok = lane < n ? w.list[pos + lane] : -1;
  }
  for (int k = 0; ok && k < my_n; ++k) {
    const int row = __shfl_sync(0xffffffffu, p.by_uid ? my_item.w : my_item.x, k - k0);
    const int pos = __shfl_sync(0xffffffffu, my_item.y, k - k0);
    const int n = __shfl_sync(0xffffffffu, my_item.z, k - k0);
    const int tok = next_tok;
    if (k + 1 < my_n) {  // prefetch the next item's record batch and tokens
      if (k + 1 - k0 == 32) {
        k0 = k + 1;
        my_item = nx_item;
        nx_item = record(k0 + 32 + lane);
      }
      const int pos1 = __shfl_sync(0xffffffffu, my_item.y, k + 1 - k0);
      const int n1 = __shfl_sync(0xffffffffu, my_item.z, k + 1 - k0);
      next_tok = lane < n1 ? w.list[pos1 + lane] : -1;
    }
    const uint32_t q = ring_slot(r, L, k);
    if (k >= pre) {
      if (bad_row(row)) break;
      ok = warp_wait(&r.empty[q], ring_parity(L, k) ^ 1u, abort, p.err);
      if (!ok) break;
      issue_rows(q, row);
    }
    uint8_t* slot = r.slots + (size_t)q * L.slot_bytes;
    if (lane == 0 && ls == nullptr) {
      const uint32_t gate_bytes = (uint32_t)n * NP * 4u;
      mbar_expect_tx(&r.full[q], gate_bytes);
      bulk_g2s(slot + L.gates_off, w.gates + (int64_t)pos * NP, gate_bytes, &r.full[q]);
    }
    // the token list (loaded one item ahead) after the copies
    if (lane < n) r.slot_tok[q * C + lane] = tok;
    if (lane == 0) r.slot_n[q] = n;
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.full[q]);
    issued = k + 1;
  }
  if (ls != nullptr) {
    // tokens with a bad id are in no work item: NaN output rows for those of
    // this CTA's slice of the batch
    const int64_t t0 = (int64_t)blockIdx.x * p.T / gridDim.x, t1 = ((int64_t)blockIdx.x + 1) * p.T / gridDim.x;
    for (int64_t t = t0 + lane; t < t1; t += 32) {
      if (__ldg(w.tok_pos + t) >= 0) continue;
      atomicOr(p.err, kErrIndex);
      float* o = p.out + t * p.D;
      for (int d = 0; d < p.D; d += 4) __stcs(reinterpret_cast<float4*>(o + d), make_float4(NAN, NAN, NAN, NAN));
    }
  }
  if (lane == 0) {  // the last copies must have landed before the CTA exits
    if (ls != nullptr) {
      mbar_drain(ls->wr_full, 0u);
      if (staged > 0) mbar_drain(ls->h_full, (uint32_t)((staged - 1) & 1));
    }
    for (int kk = issued - 1; kk >= 0 && kk >= issued - L.n_slots; --kk)
      mbar_drain(&r.full[ring_slot(r, L, kk)], ring_parity(L, kk));
  }
  __syncwarp();
}

// Consumer warps of the gather.  unit = 4 consecutive elements of D; with
// fewer units than consumer threads, Gt thread groups split the item's tokens.
// Gates: from the item's slot, or (gl != nullptr) from the CTA's gate array,
// the k-th item's at rows loff[k] ...
// A consumer thread's share of an item: units v0, v0 + vstep, ... of D / 4,
// tokens grp, grp + Gt, ... of the item.
struct UnitSplit {
  int units, Gt, grp, v0, vstep;
  bool active;
  __device__ __forceinline__ explicit UnitSplit(int D) {
    constexpr int kCT = kGroupCons * 32;
    const int lt = threadIdx.x;
    units = D >> 2;
    Gt = units >= kCT ? 1 : kCT / units;
    grp = units >= kCT ? 0 : lt / units;
    v0 = units >= kCT ? lt : lt - grp * units;
    vstep = units >= kCT ? kCT : units;
    active = grp < Gt;
  }
};

// One work item from its slot: the n tokens tok[0..n-1] with gates gs[i *
// NP ..] (this thread's units and tokens).
template <int NT, bool kExactN, bool kNf3>
__device__ __forceinline__ void combine_item(const GArgs& p, const GroupLayout& L, const UnitSplit& us,
                                             const uint8_t* slot, const float* gs, const int* tok, int n) {
  constexpr int NP = 8 * NT;
  constexpr bool kPacked = !kNf3 && NP > 16;  // 32 experts: keep rows as bf16 pairs, convert per token
  static_assert(!kNf3 || NP <= 16, "the NF3 consumer holds 16 rows");
  const int NB = p.D >> 6;
  const int units = us.units, Gt = us.Gt, grp = us.grp, v0 = us.v0, vstep = us.vstep;
  for (int v = v0; v < units; v += vstep) {
    float2 xf[kPacked ? 1 : NP][2];
    uint2 xp[kPacked ? NP : 1];
    float sc[NP];
    if constexpr (kNf3) {
      // 4 codes at bits [12u, 12u + 12) of the row's block v / 16
      const int b = v >> 4, bit = 12 * (v & 15), wi = bit >> 5, sh = bit & 31;
      const uint16_t* ss = reinterpret_cast<const uint16_t*>(slot + L.scales_off);
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        float f[4] = {0.f, 0.f, 0.f, 0.f};
        sc[j] = 0.f;
        if (kExactN || j < p.N) {
          const uint32_t* cw = reinterpret_cast<const uint32_t*>(slot + (size_t)(j * NB + b) * 24);
          const uint32_t x = __funnelshift_r(cw[wi], wi < 5 ? cw[wi + 1] : 0u, sh) & 0xfffu;
          nf3_levels4(x, f);
          sc[j] = held(__half2float(__ushort_as_half(ss[j * NB + b])));
        }
        xf[j][0] = make_float2(held(f[0]), held(f[1]));
        xf[j][1] = make_float2(held(f[2]), held(f[3]));
      }
    } else {
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        uint2 rw = make_uint2(0u, 0u);
        if (kExactN || j < p.N) rw = *reinterpret_cast<const uint2*>(slot + ((size_t)j * p.D + 4 * v) * 2);
        if (kPacked) {
          xp[kPacked ? j : 0] = rw;
        } else {
          xf[kPacked ? 0 : j][0] = make_float2(bf16_lo_held(rw.x), bf16_hi_held(rw.x));
          xf[kPacked ? 0 : j][1] = make_float2(bf16_lo_held(rw.y), bf16_hi_held(rw.y));
        }
      }
    }
    int i = grp;
    if constexpr (!kPacked) {
      // four tokens at a time (16 independent FMA chains)
      for (; i + 3 * Gt < n; i += 4 * Gt) {
        float2 o[4][2];
        if constexpr (kNf3)
          combine_quad_nf3<NP, kExactN>(xf, sc, gs + i * NP, Gt * NP, p.N, o);
        else
          combine_quad<NP, kExactN>(xf, gs + i * NP, Gt * NP, p.N, o);
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2)
          __stcs(reinterpret_cast<float4*>(p.out + (int64_t)tok[i + k2 * Gt] * p.D + 4 * v),
                 make_float4(o[k2][0].x, o[k2][0].y, o[k2][1].x, o[k2][1].y));
      }
    }
    for (; i < n; i += Gt) {
      float4 o0;
      if constexpr (kNf3)
        o0 = combine_unit_nf3<NP, kExactN>(xf, sc, gs + i * NP, p.N);
      else
        o0 = combine_unit<NP, kExactN, kPacked>(xf, xp, gs + i * NP, p.N);
      __stcs(reinterpret_cast<float4*>(p.out + (int64_t)tok[i] * p.D + 4 * v), o0);
    }
  }
}

template <int NT, bool kExactN, bool kNf3>
__device__ void ring_consumers(const GArgs& p, const GroupLayout& L, const Ring& r, int my_n,
                               const float* gl = nullptr, const int* loff = nullptr) {
  constexpr int NP = 8 * NT;
  constexpr int C = kItemTokens;
  const int lane = threadIdx.x & 31;
  volatile int* abort = r.abort;
  const UnitSplit us(p.D);
  for (int k = 0; k < my_n; ++k) {
    const uint32_t q = ring_slot(r, L, k);
    if (!warp_wait(&r.full[q], ring_parity(L, k), abort, p.err)) break;
    if (*abort) break;  // a phase completed without its item (the producer gave up)
    if (us.active) {
      const uint8_t* slot = r.slots + (size_t)q * L.slot_bytes;
      const float* gs = gl != nullptr ? gl + loff[k] * NP : reinterpret_cast<const float*>(slot + L.gates_off);
      combine_item<NT, kExactN, kNf3>(p, L, us, slot, gs, r.slot_tok + q * C, r.slot_n[q]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.empty[q]);
  }
}


template <int NT, bool kExactN, bool kNf3>
__global__ void __launch_bounds__(kGroupThreads, 1) grouped_gather_kernel(const GArgs p, const GroupWs w,
                                                                          const GroupLayout L) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Ring r = carve_ring(smem_raw, L);
  if (threadIdx.x == 0) ring_init(r, L);
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // the router's gates (and, before it, the grouping) are complete
  if (ld_relaxed_u32(&w.ctl[kCtlAbort]) != 0xFFFFFFFFu) return;  // plan abandoned (error word set)
  const int my_n = items_of_cta(w);
  if ((threadIdx.x >> 5) == kGroupProducer)
    ring_producer<8 * NT, kNf3>(p, w, L, r, my_n, nullptr);
  else
    ring_consumers<NT, kExactN, kNf3>(p, L, r, my_n);
  __syncthreads();
}

// ---- CTA-local layer kernel: router and gather in one launch ----
//
// One CTA per SM, no waits on other CTAs.  The CTA's share of the grouping
// (group_share_kernel) lists its work items in processing order and their
// tokens.  The consumer warps compute those tokens' gates, two 16-token tiles
// at a time -- A fragments loaded from h by token id, B fragments from Wr
// (one bulk copy into the ring's last slot) by ldmatrix, mma.sync with the
// router kernels' k-step split, k-slot order and partial-sum order, then
// their softmax, so the gates are bit-identical to theirs -- into a gate array
// in shared memory, and then combine as in grouped_gather_kernel, reading
// each item's gates from that array.  Meanwhile the producer warp has
// requested the row blocks of the first items (Wr's slot once the MMAs are
// done).

constexpr int kFusedKB = 16;  // k-steps per warp (D <= 2048)

// Barrier over the 8 consumer warps only (the producer warp runs apart).
struct ConsumerSync {
  __device__ __forceinline__ void operator()() const {
    asm volatile("bar.sync 1, %0;" ::"n"(kGroupCons * 32) : "memory");
  }
};

// B fragments of k-step ks for both 8-expert halves from Wr as copied
// ([D][N] bf16, N = 8 NT): one ldmatrix.trans of 2 NT 8x8 blocks, each
// lane giving the address of one row, in the router kernels' k-slot order
// (slots 2c, 2c+1 <- d = 4c, 4c+1; slots 2c+8, 2c+9 <- d = 4c+2, 4c+3).
template <int NT>
__device__ __forceinline__ void wr_fragments(uint2 (&b)[NT], const uint16_t* wr_s, int ks) {
  const int lane = threadIdx.x & 31;
  const int m = lane >> 3, rr = lane & 7;  // matrix m = (slot half m & 1, expert half m >> 1); its row rr
  const int slot = rr + 8 * (m & 1);
  const int dl = slot < 8 ? 4 * (slot >> 1) + (slot & 1) : 4 * ((slot - 8) >> 1) + 2 + (slot & 1);
  const uint32_t addr = smem_u32(wr_s + (ks * 16 + dl) * (8 * NT) + 8 * ((m >> 1) & (NT - 1)));
  if constexpr (NT == 2) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(b[0].x), "=r"(b[0].y), "=r"(b[1].x), "=r"(b[1].y)
                 : "r"(addr));
  } else {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(b[0].x), "=r"(b[0].y)
                 : "r"(addr));
  }
}

// B fragments of k-step ks (both 8-expert halves) from Wr as copied, for
// any N <= NP: element loads, zero past N.
template <int NT>
__device__ __forceinline__ void wr_fragments_any(uint2 (&b)[NT], const uint16_t* wr_s, int ks, int N) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int j = nt * 8 + g;
    uint32_t e[4] = {0u, 0u, 0u, 0u};
    if (j < N) {
      const uint16_t* src = wr_s + (ks * 16 + 4 * c) * N + j;
#pragma unroll
      for (int u = 0; u < 4; ++u) e[u] = src[u * N];
    }
    b[nt] = make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
  }
}

// Waits of the consumer warps on a barrier of the router phase, with one
// verdict for all of them (the tile loop holds barriers, so every warp must
// take the same path): a warp whose wait failed says so before the barrier
// and all read the verdict after it.
__device__ __forceinline__ bool consumers_wait(uint64_t* b, uint32_t parity, volatile int* abort, unsigned* err,
                                               volatile int* fail) {
  if (!warp_wait(b, parity, abort, err) && (threadIdx.x & 31) == 0) *fail = 1;
  ConsumerSync{}();
  return *fail == 0;
}

// Router scratch of the local kernel: two tiles finished together.
constexpr int kPairRows = 2 * kTileMax;

template <int NP>
__host__ __device__ constexpr size_t pair_scratch_bytes() {
  return (size_t)kWarps * kPairRows * NP * 4;  // the partial sums (the gates go elsewhere)
}

struct PairScratch {
  float* part;   // [kWarps][kPairRows][NP] partial logits
  float* gates;  // [kPairRows][NP]
  int* tok;      // [kPairRows] list positions
};

// This warp's partial logits of one tile -> rows row0 .. row0+15.
template <int NT>
__device__ __forceinline__ void pair_store_partials(const PairScratch& ps, const float (&acc)[NT][4], int row0) {
  constexpr int NP = 8 * NT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  float* pw = ps.part + warp * kPairRows * NP;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    pw[(row0 + g) * NP + nt * 8 + 2 * c] = acc[nt][0];
    pw[(row0 + g) * NP + nt * 8 + 2 * c + 1] = acc[nt][1];
    pw[(row0 + g + 8) * NP + nt * 8 + 2 * c] = acc[nt][2];
    pw[(row0 + g + 8) * NP + nt * 8 + 2 * c + 1] = acc[nt][3];
  }
}

// Sum of the partial logits (warps in order), max-subtracted softmax over
// the N experts: the arithmetic of router_softmax, row for row.
template <int NT>
__device__ __forceinline__ void pair_softmax(const PairScratch& ps, int rows, int N) {
  constexpr int NP = 8 * NT;
  constexpr int RPW = 32 / NP;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / NP, jl = lane % NP;
  for (int rb = warp * RPW; rb < rows; rb += kWarps * RPW) {
    const int r = rb + sub;
    const bool act = r < rows;
    float z = 0.f;
    if (act) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) z += ps.part[(w * kPairRows + r) * NP + jl];
    }
    const bool valid = act && jl < N;
    float m = valid ? z : -INFINITY;
#pragma unroll
    for (int off = NP / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float e = valid ? expf(z - m) : 0.f;
    float sum = e;
#pragma unroll
    for (int off = NP / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (act) ps.gates[r * NP + jl] = valid ? e / sum : 0.f;
  }
}

// A fragments of a tile whose row rr is token tok[rr] (rr < rows; rows past
// read as zero), in router_load_a's k-slot order.
template <int KB>
__device__ __forceinline__ void router_load_a_rows(RouterA<KB>& A, const uint16_t* __restrict__ h, const int* tok,
                                                   int rows, int D, int kb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const bool ok0 = g < rows, ok1 = g + 8 < rows;
  const uint16_t* h0 = h + (int64_t)(ok0 ? __ldg(tok + g) : 0) * D + 4 * c;
  const uint16_t* h1 = h + (int64_t)(ok1 ? __ldg(tok + g + 8) : 0) * D + 4 * c;
  const int ksteps = D >> 4;
#pragma unroll
  for (int i = 0; i < KB; ++i) {
    const int ks = kb + i * kWarps;
    const bool in = ks < ksteps;
    A.a0[i] = (in && ok0) ? __ldg(reinterpret_cast<const uint2*>(h0 + (ks << 4))) : make_uint2(0u, 0u);
    A.a1[i] = (in && ok1) ? __ldg(reinterpret_cast<const uint2*>(h1 + (ks << 4))) : make_uint2(0u, 0u);
  }
}

// A fragments of a staged router tile (row rr at stage + rr * pitch, rr <
// rows; rows past read as zero), in router_load_a's k-slot order.  With
// pitch = 2 D + 32 the 32 lanes of one load hit every bank pair once.
template <int KB>
__device__ __forceinline__ void router_load_a_smem(RouterA<KB>& A, const uint8_t* stage, int pitch, int rows, int D,
                                                   int kb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const bool ok0 = g < rows, ok1 = g + 8 < rows;
  const uint8_t* r0 = stage + (size_t)g * pitch + 8 * c;
  const uint8_t* r1 = stage + (size_t)(g + 8) * pitch + 8 * c;
  const int ksteps = D >> 4;
#pragma unroll
  for (int i = 0; i < KB; ++i) {
    const int ks = kb + i * kWarps;
    const bool in = ks < ksteps;
    A.a0[i] = (in && ok0) ? *reinterpret_cast<const uint2*>(r0 + ks * 32) : make_uint2(0u, 0u);
    A.a1[i] = (in && ok1) ? *reinterpret_cast<const uint2*>(r1 + ks * 32) : make_uint2(0u, 0u);
  }
}

// Consumer warps: the gates of the CTA's n_tok listed tokens (tok[i]) into
// gl[n_tok][NP].  Each warp takes the B fragments of its k-steps into
// registers as soon as Wr lands and Wr's slots go back to the ring.  A
// fragments: from the staging slots, tile by tile as the producer's bulk
// copies land (each tile's slots released after its MMAs); without staging
// slots, from h by token id, the next tile's right after the current tile's
// MMAs.  Two tiles share one partial-sum exchange and softmax.  Returns
// false (uniformly) if a copy never arrived.
template <int NT, bool kExactN>
__device__ bool local_router_phase(const GArgs& p, const PairScratch& ps, const uint16_t* wr_s, const uint8_t* stage,
                                   const LocalSync& ls, const int* tok, int n_tok, float* gl, volatile int* abort,
                                   volatile int* fail) {
  constexpr int KB = kFusedKB;
  constexpr int NP = 8 * NT;
  const int warp = threadIdx.x >> 5;
  const int ksteps = p.D >> 4;
  const int n_tiles = (n_tok + kTileMax - 1) / kTileMax;
  const bool staged = ls.n_st > 0;
  auto rows_of = [&](int t) {
    const int left = n_tok - t * kTileMax;
    return left < 0 ? 0 : (left < kTileMax ? left : kTileMax);
  };
  RouterA<KB> A;
  if (!staged && n_tiles > 0) router_load_a_rows<KB>(A, p.h, tok, rows_of(0), p.D, warp);
  const bool ok = consumers_wait(ls.wr_full, 0u, abort, p.err, fail);
  // B fragments of k-steps warp + 8i, in the router kernels' k-slot order
  uint2 bw[KB][NT];
#pragma unroll
  for (int i = 0; i < KB; ++i) {
    const int ks = warp + i * kWarps;
    if (ok && ks < ksteps) {
      if (kExactN && p.N == NP)
        wr_fragments<NT>(bw[i], wr_s, ks);
      else
        wr_fragments_any<NT>(bw[i], wr_s, ks, p.N);
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) bw[i][nt] = make_uint2(0u, 0u);
    }
  }
  ConsumerSync{}();
  if (ok && threadIdx.x == 0) mbar_arrive(ls.wr_free);  // Wr's slots go back to the ring
  if (!ok) return false;
  auto mma_tile = [&](float (&acc)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int i = 0; i < KB; ++i) {
      if (warp + i * kWarps < ksteps) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816(acc[nt], A.a0[i].x, A.a1[i].x, A.a0[i].y, A.a1[i].y, bw[i][nt].x, bw[i][nt].y);
      }
    }
  };
  // tile t's MMAs into acc: a staged tile waits for its copies and releases
  // the staging slots after its MMAs (every warp past them); otherwise the
  // next tile's A fragments are requested right after
  auto tile = [&](int t, float (&acc)[NT][4]) {
    if (staged) {
      if (!consumers_wait(ls.h_full, (uint32_t)(t & 1), abort, p.err, fail)) return false;
      router_load_a_smem<KB>(A, stage, ls.pitch, rows_of(t), p.D, warp);
      mma_tile(acc);
      ConsumerSync{}();
      if (threadIdx.x == 0) mbar_arrive(ls.h_empty);
    } else {
      mma_tile(acc);
      if (t + 1 < n_tiles) router_load_a_rows<KB>(A, p.h, tok + (t + 1) * kTileMax, rows_of(t + 1), p.D, warp);
    }
    return true;
  };
  for (int t = 0; t < n_tiles; t += 2) {
    float acc[NT][4];
    if (!tile(t, acc)) return false;
    pair_store_partials<NT>(ps, acc, 0);
    if (t + 1 < n_tiles) {
      if (!tile(t + 1, acc)) return false;
      pair_store_partials<NT>(ps, acc, kTileMax);
    }
    ConsumerSync{}();
    PairScratch pg = ps;
    pg.gates = gl + (size_t)t * kTileMax * NP;
    pair_softmax<NT>(pg, rows_of(t) + rows_of(t + 1), p.N);
    ConsumerSync{}();
  }
  return true;
}

constexpr uint32_t kWrChunk = 4096;  // bytes per bulk copy of Wr

template <int NT, bool kExactN, bool kNf3>
__global__ void __launch_bounds__(kGroupThreads, 1) grouped_local_kernel(const GArgs p, const GroupWs w,
                                                                         const GroupLayout L, int scap) {
  constexpr int NP = 8 * NT;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Ring r = carve_ring(smem_raw, L);
  uint8_t* scratch = smem_raw + (ring_bytes(L.n_slots, L.slot_bytes) + 127) / 128 * 128;
  const PairScratch ps{reinterpret_cast<float*>(scratch), nullptr, nullptr};       // partial sums
  float* gl = reinterpret_cast<float*>(scratch + (size_t)kWarps * kPairRows * NP * 4);  // [scap][NP] gates
  int* loff = reinterpret_cast<int*>(gl + (size_t)scap * NP);                       // [scap + 1]
  __shared__ int skip_s, fail_s;
  __shared__ __align__(8) uint64_t bars[4];
  const int b = blockIdx.x, lane = threadIdx.x & 31;
  const bool producer = (threadIdx.x >> 5) == kGroupProducer;
  const int wr_slot0 = L.n_slots - wr_slots(L, p.N, p.D);
  uint8_t* wr_slot = r.slots + (size_t)wr_slot0 * L.slot_bytes;
  const int* tok = w.share_tok + (size_t)b * scap;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    ring_init(r, L, 2);  // full: the row block's copies, the token list
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // the grouping and every earlier kernel are complete
  if (producer) {
    // Wr first (the router phase waits for it), in chunks taken in a
    // CTA-dependent order so that the CTAs' requests spread over L2
    const uint32_t wr_bytes = (uint32_t)p.N * (uint32_t)p.D * 2u;
    const uint32_t n_ch = (wr_bytes + kWrChunk - 1) / kWrChunk;  // <= 16 (N <= 16, D <= 2048)
    if (lane == 0) mbar_expect_tx(&bars[0], wr_bytes);
    __syncwarp();
    if ((uint32_t)lane < n_ch) {
      const uint32_t off = ((lane + (uint32_t)b) % n_ch) * kWrChunk;
      bulk_g2s(wr_slot + off, reinterpret_cast<const uint8_t*>(p.Wr) + off,
               wr_bytes - off < kWrChunk ? wr_bytes - off : kWrChunk, &bars[0]);
    }
  }
  // the CTA's counts (all threads), the token ids of the first router tile
  // (producer lanes 0-15; scap >= 32), the control words (thread 0)
  const int2 sn = reinterpret_cast<const int2*>(w.share_n)[b];
  const int tok0 = producer && lane < kTileMax ? __ldg(tok + lane) : 0;
  if (threadIdx.x == 0) {
    const unsigned ab = ld_relaxed_u32(&w.ctl[kCtlAbort]), grid = ld_relaxed_u32(&w.ctl[kCtlShareGrid]);
    // plan abandoned (error word set): skip; shares for another CTA count: error
    skip_s = ab != 0xFFFFFFFFu ? 1 : (grid != gridDim.x || sn.x < 0 || sn.y < 0 || sn.x > scap || sn.y > scap) ? 2 : 0;
    if (skip_s == 2) atomicOr(p.err, kErrGrouping);
    fail_s = 0;
  }
  __syncthreads();
  if (skip_s) {
    if (producer && lane == 0) mbar_drain(&bars[0], 0u);
    return;
  }
  const int my_n = sn.x, n_tok = sn.y;
  // staging slots for the router tiles: those before Wr's that hold 16 h
  // rows, if at least one slot is left for row blocks
  const int pitch = 2 * p.D + 32;
  const int st_n = (int)(((int64_t)kTileMax * pitch + L.slot_bytes - 1) / L.slot_bytes);
  const int st_slot0 = wr_slot0 - st_n >= 1 ? wr_slot0 - st_n : wr_slot0;
  const LocalSync ls{&bars[0], &bars[1], &bars[2], &bars[3], w.share_rec + (size_t)b * scap, tok, wr_slot0, st_slot0,
                     st_slot0 < wr_slot0 ? (n_tok + kTileMax - 1) / kTileMax : 0, n_tok, pitch};
  if (producer) {
    ring_producer<NP, kNf3>(p, w, L, r, my_n, &ls, tok0);
  } else {
    // step offsets into shared memory (my_n <= scap < the consumer threads);
    // the router phase's first barrier orders them before their readers
    if ((int)threadIdx.x <= my_n) loff[threadIdx.x] = __ldg(w.share_off + (size_t)b * (scap + 1) + threadIdx.x);
    const bool ok = local_router_phase<NT, kExactN>(p, ps, reinterpret_cast<const uint16_t*>(wr_slot),
                                                    r.slots + (size_t)st_slot0 * L.slot_bytes, ls, tok, n_tok, gl,
                                                    r.abort, &fail_s);
    if (!ok && threadIdx.x == 0) *r.abort = 1;  // the producer stops too
    ring_consumers<NT, kExactN, kNf3>(p, L, r, ok ? my_n : 0, gl, loff);
  }
  __syncthreads();
}

// ---- Interleaved layer kernel: router tiles and work items in one ring ----
//
// One CTA per SM on the grouping's shares, like the CTA-local kernel, but its
// ring carries two kinds of entries in one order: a router tile (the h rows
// of 16 consecutive tokens of the share, one bulk copy per row, pitch bytes
// apart) and a work item (the id's row block).  A tile goes in just before
// the first item with a token in it, so h and the row blocks stream from
// memory together and an item's gates are computed right before it is
// combined, instead of in a router pass over the whole share first.  Wr
// arrives once, in the ring's last slot, and stays in registers as each
// consumer warp's B fragments; the slot then joins the ring.  The gates
// (same mma.sync k-step split, k-slot order, partial-sum order and softmax as
// the router kernels) go to a gate array in shared memory; the combine is
// that of grouped_gather_kernel.

struct StreamSync {
  uint64_t* wr_full;  // Wr's copies landed
  uint64_t* wr_free;  // every consumer warp holds its B fragments
  const int4* recs;   // the CTA's item records (global memory), processing order
  const int* loff;    // [my_n + 1] token offset of each item in the share (shared memory)
  const int* tok;     // [n_tok] the share's tokens (shared memory)
  int my_n, n_tok, n_tiles, pitch, wr_slot;
};

// Whether the next ring entry, with t tiles and k items before it, is tile
// t: while a tile holds a token of item k (or of an earlier one).  Once all
// items are placed, all tiles are (the last item ends at n_tok).
__device__ __forceinline__ bool stream_tile_next(const StreamSync& ss, int t, int k) {
  return t < ss.n_tiles && t * kTileMax < ss.loff[k + 1];
}

// Producer warp of the interleaved kernel: entry e into slot e mod n_slots
// once its previous entry is consumed (in the first lap at once, Wr's slot
// once the B fragments are in registers); a tile's rows by its lanes, an
// item's row block by lane 0.  Item records are read 32 at a time.
template <int NP>
__device__ void stream_producer(const GArgs& p, const GroupWs& w, const GroupLayout& L, const Ring& r,
                                const StreamSync& ss) {
  const int lane = threadIdx.x & 31;
  volatile int* abort = r.abort;
  const uint32_t row_bytes = (uint32_t)p.N * (uint32_t)p.D * 2u, h_row = (uint32_t)p.D * 2u;
  const int n_entries = ss.n_tiles + ss.my_n;
  const int4 none = make_int4(0, 0, 0, 0);
  int t = 0, k = 0, k0 = 0, issued = 0;
  int4 rec = lane < ss.my_n ? ss.recs[lane] : none;
  for (int e = 0; e < n_entries; ++e) {
    const uint32_t q = ring_slot(r, L, e);
    bool ok = true;
    if (e >= L.n_slots)
      ok = warp_wait(&r.empty[q], ring_parity(L, e) ^ 1u, abort, p.err);
    else if ((int)q == ss.wr_slot)
      ok = warp_wait(ss.wr_free, 0u, abort, p.err);
    if (!ok) break;
    uint8_t* slot = r.slots + (size_t)q * L.slot_bytes;
    if (stream_tile_next(ss, t, k)) {
      const int rows = ss.n_tok - t * kTileMax < kTileMax ? ss.n_tok - t * kTileMax : kTileMax;
      if (lane == 0) mbar_expect_tx(&r.full[q], (uint32_t)rows * h_row);
      __syncwarp();
      if (lane < rows)
        bulk_g2s(slot + (size_t)lane * ss.pitch, p.h + (int64_t)ss.tok[t * kTileMax + lane] * p.D, h_row, &r.full[q]);
      ++t;
    } else {
      if (k - k0 == 32) {
        k0 = k;
        rec = k0 + lane < ss.my_n ? ss.recs[k0 + lane] : none;
      }
      const int row = __shfl_sync(0xffffffffu, p.by_uid ? rec.w : rec.x, k - k0);
      if (p.by_uid && (int64_t)row >= p.rows) {  // staging buffer smaller than the batch's distinct ids
        if (lane == 0) atomicOr(p.err, kErrIndex);
        *abort = 1;
        break;
      }
      if (lane == 0) {
        mbar_expect_tx(&r.full[q], row_bytes);
        bulk_g2s(slot, p.table + (int64_t)row * p.N * p.D, row_bytes, &r.full[q]);
      }
      ++k;
    }
    issued = e + 1;
  }
  // tokens with a bad id are in no work item: NaN output rows for those of
  // this CTA's slice of the batch
  const int64_t t0 = (int64_t)blockIdx.x * p.T / gridDim.x, t1 = ((int64_t)blockIdx.x + 1) * p.T / gridDim.x;
  for (int64_t tt = t0 + lane; tt < t1; tt += 32) {
    if (__ldg(w.tok_pos + tt) >= 0) continue;
    atomicOr(p.err, kErrIndex);
    float* o = p.out + tt * p.D;
    for (int d = 0; d < p.D; d += 4) __stcs(reinterpret_cast<float4*>(o + d), make_float4(NAN, NAN, NAN, NAN));
  }
  if (lane == 0) {  // the last copies must have landed before the CTA exits
    mbar_drain(ss.wr_full, 0u);
    for (int e = issued - 1; e >= 0 && e >= issued - L.n_slots; --e)
      mbar_drain(&r.full[ring_slot(r, L, e)], ring_parity(L, e));
  }
  __syncwarp();
}

// Consumer warps of the interleaved kernel.  A tile: A fragments from the
// slot (then the slot is released), MMAs against the held B fragments,
// partial sums exchanged, softmax into the gate array -- every consumer
// warp takes part, so tile waits give one verdict for all.  An item: the
// combine of ring_consumers with the gates from the gate array.  A warp whose
// item wait failed skips the remaining items but still meets the other warps
// at the next tile, where all of them stop.
template <int NT, bool kExactN>
__device__ void stream_consumers(const GArgs& p, const GroupLayout& L, const Ring& r, const StreamSync& ss,
                                 const PairScratch& ps, float* gl, const uint16_t* wr_s, volatile int* fail) {
  constexpr int KB = kFusedKB;
  constexpr int NP = 8 * NT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ksteps = p.D >> 4;
  volatile int* abort = r.abort;
  const bool ok = consumers_wait(ss.wr_full, 0u, abort, p.err, fail);
  // B fragments of k-steps warp + 8i, in the router kernels' k-slot order
  uint2 bw[KB][NT];
#pragma unroll
  for (int i = 0; i < KB; ++i) {
    const int ks = warp + i * kWarps;
    if (ok && ks < ksteps) {
      if (kExactN && p.N == NP)
        wr_fragments<NT>(bw[i], wr_s, ks);
      else
        wr_fragments_any<NT>(bw[i], wr_s, ks, p.N);
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) bw[i][nt] = make_uint2(0u, 0u);
    }
  }
  ConsumerSync{}();
  if (ok && threadIdx.x == 0) mbar_arrive(ss.wr_free);  // Wr's slot goes back to the ring
  if (!ok) return;
  const UnitSplit us(p.D);
  const int n_entries = ss.n_tiles + ss.my_n;
  int t = 0, k = 0;
  bool dead = false;
  for (int e = 0; e < n_entries; ++e) {
    const uint32_t q = ring_slot(r, L, e), par = ring_parity(L, e);
    const uint8_t* slot = r.slots + (size_t)q * L.slot_bytes;
    if (stream_tile_next(ss, t, k)) {
      if (!consumers_wait(&r.full[q], par, abort, p.err, fail)) return;
      const int rows = ss.n_tok - t * kTileMax < kTileMax ? ss.n_tok - t * kTileMax : kTileMax;
      RouterA<KB> A;
      router_load_a_smem<KB>(A, slot, ss.pitch, rows, p.D, warp);
      __syncwarp();
      if (lane == 0) mbar_arrive(&r.empty[q]);
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
      for (int i = 0; i < KB; ++i) {
        if (warp + i * kWarps < ksteps) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_16816(acc[nt], A.a0[i].x, A.a1[i].x, A.a0[i].y, A.a1[i].y, bw[i][nt].x, bw[i][nt].y);
        }
      }
      pair_store_partials<NT>(ps, acc, 0);
      ConsumerSync{}();
      PairScratch pg = ps;
      pg.gates = gl + (size_t)t * kTileMax * NP;
      pair_softmax<NT>(pg, rows, p.N);
      ConsumerSync{}();
      ++t;
    } else {
      if (!dead) {
        dead = !warp_wait(&r.full[q], par, abort, p.err);
        if (!dead && us.active) {
          const int o = ss.loff[k];
          combine_item<NT, kExactN, false>(p, L, us, slot, gl + (size_t)o * NP, ss.tok + o, ss.loff[k + 1] - o);
        }
        __syncwarp();
        if (lane == 0) {
          if (dead)
            *fail = 1;
          else
            mbar_arrive(&r.empty[q]);
        }
      }
      ++k;
    }
  }
}

template <int NT, bool kExactN>
__global__ void __launch_bounds__(kGroupThreads, 1) grouped_stream_kernel(const GArgs p, const GroupWs w,
                                                                          const GroupLayout L, int scap, int pitch) {
  constexpr int NP = 8 * NT;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Ring r = carve_ring(smem_raw, L);
  uint8_t* scratch = smem_raw + (ring_bytes(L.n_slots, L.slot_bytes) + 127) / 128 * 128;
  const PairScratch ps{reinterpret_cast<float*>(scratch), nullptr, nullptr};  // partial sums
  float* gl = reinterpret_cast<float*>(scratch + pair_scratch_bytes<NP>());    // [scap][NP] gates
  int* loff = reinterpret_cast<int*>(gl + (size_t)scap * NP);                   // [scap + 1]
  int* tok_s = loff + scap + 1;                                                 // [scap]
  __shared__ int skip_s, fail_s;
  __shared__ __align__(8) uint64_t bars[2];
  const int b = blockIdx.x, lane = threadIdx.x & 31;
  const bool producer = (threadIdx.x >> 5) == kGroupProducer;
  const int wr_slot = L.n_slots - 1;
  uint8_t* wr_p = r.slots + (size_t)wr_slot * L.slot_bytes;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    ring_init(r, L, 1);  // full: one arrival, with the entry's copy bytes
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // the grouping and every earlier kernel are complete
  if (producer) {
    // Wr (one slot), in chunks taken in a CTA-dependent order so that the
    // CTAs' requests spread over L2
    const uint32_t wr_bytes = (uint32_t)p.N * (uint32_t)p.D * 2u;
    const uint32_t n_ch = (wr_bytes + kWrChunk - 1) / kWrChunk;  // <= 16 (N <= 16, D <= 2048)
    if (lane == 0) mbar_expect_tx(&bars[0], wr_bytes);
    __syncwarp();
    if ((uint32_t)lane < n_ch) {
      const uint32_t off = ((lane + (uint32_t)b) % n_ch) * kWrChunk;
      bulk_g2s(wr_p + off, reinterpret_cast<const uint8_t*>(p.Wr) + off,
               wr_bytes - off < kWrChunk ? wr_bytes - off : kWrChunk, &bars[0]);
    }
  }
  const int2 sn = reinterpret_cast<const int2*>(w.share_n)[b];
  if (threadIdx.x == 0) {
    const unsigned ab = ld_relaxed_u32(&w.ctl[kCtlAbort]), grid = ld_relaxed_u32(&w.ctl[kCtlShareGrid]);
    // plan abandoned (error word set): skip; shares for another CTA count: error
    skip_s = ab != 0xFFFFFFFFu ? 1 : (grid != gridDim.x || sn.x < 0 || sn.y < 0 || sn.x > scap || sn.y > scap) ? 2 : 0;
    if (skip_s == 2) atomicOr(p.err, kErrGrouping);
    fail_s = 0;
  }
  __syncthreads();
  if (skip_s) {
    if (producer && lane == 0) mbar_drain(&bars[0], 0u);
    return;
  }
  const int my_n = sn.x, n_tok = sn.y;
  // the share's item offsets and tokens into shared memory
  for (int i = threadIdx.x; i <= my_n; i += kGroupThreads) loff[i] = __ldg(w.share_off + (size_t)b * (scap + 1) + i);
  for (int i = threadIdx.x; i < n_tok; i += kGroupThreads) tok_s[i] = __ldg(w.share_tok + (size_t)b * scap + i);
  __syncthreads();
  const StreamSync ss{&bars[0], &bars[1], w.share_rec + (size_t)b * scap, loff, tok_s, my_n, n_tok,
                      (n_tok + kTileMax - 1) / kTileMax, pitch, wr_slot};
  if (producer)
    stream_producer<NP>(p, w, L, r, ss);
  else
    stream_consumers<NT, kExactN>(p, L, r, ss, ps, gl, reinterpret_cast<const uint16_t*>(wr_p), &fail_s);
  __syncthreads();
}

// Ring slot of a work item: the id's row block (bf16 table: N rows of D;
// NF3 table: N x D/64 24-byte code blocks, then the fp16 scales at
// scales_off), then the gates of up to kItemTokens tokens at gates_off.
template <int NT>
GroupLayout group_layout(int N, int D, bool nf3) {
  constexpr int NP = 8 * NT;
  GroupLayout L{};
  int64_t off;
  if (nf3) {
    const int64_t NB = D / 64;
    L.scales_off = (int)((N * NB * 24 + 127) / 128 * 128);
    off = L.scales_off + N * NB * 2;
  } else {
    off = (int64_t)N * D * 2;
  }
  L.gates_off = (int)((off + 127) / 128 * 128);
  L.slot_bytes = (int)((L.gates_off + (int64_t)kItemTokens * NP * 4 + 127) / 128 * 128);
  L.n_slots = (int)std::min<int64_t>(16, kRingBudget / L.slot_bytes);
  return L;
}


// The CTA-local layer kernel (bf16 or NF3 table, N <= 16, D <= 2048: a
// warp's k-steps fit kFusedKB), one CTA per SM, on the grouping's shares
// (built for this SM count when share_cap < kShareCapLimit).
template <int NT, bool kExactN, bool kNf3>
mole_status launch_local(const GArgs& p, const GroupWs& w, cudaStream_t stream) {
  constexpr int NP = 8 * NT;
  static_assert(NT <= 2, "the router phase holds B fragments of at most 16 experts");
  // (the staged router tiles are bulk copies of h rows: 16-byte aligned rows)
  if (p.D > 16 * kWarps * kFusedKB || !aligned16(p.Wr) || !aligned16(p.h) || p.D % 8 != 0)
    return MOLE_ERR_UNSUPPORTED;
  const GroupLayout L = group_layout<NT>(p.N, p.D, kNf3);
  if (L.n_slots < 2 || wr_slots(L, p.N, (int)p.D) >= L.n_slots) return MOLE_ERR_UNSUPPORTED;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  if (!shares_apply(p.T, n_sm)) return MOLE_ERR_UNSUPPORTED;
  const int64_t scap = share_cap(p.T, n_sm);
  static_assert(kShareCapLimit <= kGroupCons * 32, "a consumer thread per step offset");
  const size_t smem = (ring_bytes(L.n_slots, L.slot_bytes) + 127) / 128 * 128 + pair_scratch_bytes<NP>() +
                      (size_t)scap * NP * 4 + (size_t)(scap + 1) * 4;
  if (smem > 227 * 1024) return MOLE_ERR_UNSUPPORTED;
  auto kern = grouped_local_kernel<NT, kExactN, kNf3>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOLE_ERR_CUDA;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGroupThreads, smem) != cudaSuccess || occ < 1)
    return MOLE_ERR_UNSUPPORTED;
  return cuda_status(launch_pdl(kern, (unsigned)n_sm, kGroupThreads, smem, stream, p, w, L, (int)scap));
}

// The interleaved layer kernel (bf16 table, N <= 16, D <= 2048), one CTA
// per SM, on the grouping's shares.  Slots hold a row block or a 16-row
// router tile, whichever is larger; at least three of them.
template <int NT, bool kExactN>
mole_status launch_stream(const GArgs& p, const GroupWs& w, cudaStream_t stream) {
  constexpr int NP = 8 * NT;
  if (p.D > 16 * kWarps * kFusedKB || !aligned16(p.Wr) || !aligned16(p.h) || p.D % 8 != 0)
    return MOLE_ERR_UNSUPPORTED;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  if (!shares_apply(p.T, n_sm)) return MOLE_ERR_UNSUPPORTED;
  const int64_t scap = share_cap(p.T, n_sm);
  const int pitch = 2 * p.D + 32;
  GroupLayout L{};
  const int64_t need = std::max<int64_t>((int64_t)p.N * p.D * 2, (int64_t)kTileMax * pitch);
  L.slot_bytes = (int)((need + 127) / 128 * 128);
  L.gates_off = L.slot_bytes;
  const size_t fixed = pair_scratch_bytes<NP>() + (size_t)scap * NP * 4 + (size_t)(2 * scap + 1) * 4;
  constexpr size_t kMax = 227 * 1024 - 256;  // (the static barriers and flags)
  int n = 16;
  while (n >= 3 && (ring_bytes(n, L.slot_bytes) + 127) / 128 * 128 + fixed > kMax) --n;
  if (n < 3) return MOLE_ERR_UNSUPPORTED;
  L.n_slots = n;
  const size_t smem = (ring_bytes(n, L.slot_bytes) + 127) / 128 * 128 + fixed;
  auto kern = grouped_stream_kernel<NT, kExactN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOLE_ERR_CUDA;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGroupThreads, smem) != cudaSuccess || occ < 1)
    return MOLE_ERR_UNSUPPORTED;
  return cuda_status(launch_pdl(kern, (unsigned)n_sm, kGroupThreads, smem, stream, p, w, L, (int)scap, pitch));
}

// Batches from about 3/4 of a 128-token tile per SM up take the interleaved
// kernel; below that the CTA-local kernel's router pass over its share is
// short (at 4096 tokens on 148 SMs, two tiles) and it is as fast.
bool stream_preferred(int64_t T) {
  const int n_sm = num_sms();
  return n_sm > 0 && (T + 127) / 128 >= (int64_t)n_sm * 3 / 4;
}

// Kernel choice per layer call.  bf16 table: the interleaved kernel (large
// batches) or the CTA-local kernel, else the mma.sync router kernel + gather
// -- every bf16 path computes its gates with the mma.sync router arithmetic,
// so grouped and ungrouped calls agree bit for bit.  NF3 table: the
// CTA-local kernel below the tensor-core router's size, else that router
// (as the ungrouped NF3 call) + gather.
template <int NT, bool kExactN, bool kNf3>
mole_status launch_layer(const GArgs& p, const GroupWs& w, cudaStream_t stream) {
  constexpr int NP = 8 * NT;
  const bool tc_router = kNf3 && router_tc_supported(p.T, p.N, p.D, p.h, p.Wr);
  if constexpr (NT <= 2) {
    if (!kNf3 && stream_preferred(p.T)) {
      const mole_status st = launch_stream<NT, kExactN>(p, w, stream);
      if (st != MOLE_ERR_UNSUPPORTED) return st;
    }
    if (!tc_router) {
      const mole_status st = launch_local<NT, kExactN, kNf3>(p, w, stream);
      if (st != MOLE_ERR_UNSUPPORTED) return st;
    }
  }
  const GroupLayout L = group_layout<NT>(p.N, p.D, kNf3);
  if (L.n_slots < 2) return MOLE_ERR_UNSUPPORTED;
  const size_t gsmem = ring_bytes(L.n_slots, L.slot_bytes);
  const size_t rsmem = smem_bytes_for<true, NP>(p.D);
  if (gsmem > 227 * 1024 || rsmem > 227 * 1024) return MOLE_ERR_UNSUPPORTED;
  auto rkern = router_group_kernel<NT>;
  auto gkern = grouped_gather_kernel<NT, kExactN, kNf3>;
  if (cudaFuncSetAttribute(rkern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem) != cudaSuccess ||
      cudaFuncSetAttribute(gkern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem) != cudaSuccess)
    return MOLE_ERR_CUDA;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rkern, kThreads, rsmem) != cudaSuccess || occ < 1)
    return MOLE_ERR_UNSUPPORTED;
  const int64_t n_tiles = (p.T + kTileMax - 1) / kTileMax;
  if (tc_router) {
    const mole_status st = router_tc_launch(p.h, p.Wr, p.T, p.D, true, p.out, w.tok_pos, w.gates, stream);
    if (st != MOLE_OK) return st;
  } else if (launch_pdl(rkern, (unsigned)std::min<int64_t>(n_tiles, (int64_t)occ * n_sm), kThreads, rsmem, stream,
                        p, w) != cudaSuccess) {
    return MOLE_ERR_CUDA;
  }
  if (launch_pdl(gkern, (unsigned)n_sm, kGroupThreads, gsmem, stream, p, w, L) != cudaSuccess) return MOLE_ERR_CUDA;
  return MOLE_OK;
}

template <bool kNf3>
mole_status layer_dispatch(const GArgs& p, const GroupWs& w, cudaStream_t stream) {
  if (p.N == 16) return launch_layer<2, true, kNf3>(p, w, stream);
  if (p.N == 8) return launch_layer<1, true, kNf3>(p, w, stream);
  if (p.N < 8) return launch_layer<1, false, kNf3>(p, w, stream);
  if (p.N < 16) return launch_layer<2, false, kNf3>(p, w, stream);
  if (kNf3) return MOLE_ERR_UNSUPPORTED;  // the NF3 consumer holds at most 16 rows
  if (p.N == 32) return launch_layer<4, true, false>(p, w, stream);
  return launch_layer<4, false, false>(p, w, stream);
}

// Whether the grouped kernels take a call of this shape (else the
// mole_lookup_combine kernels do, and the grouping is not used).
bool grouped_applies(int64_t T, int N, int D, bool nf3) {
  if (T < kGroupedMinT || T > kGroupedMaxT || N < 1 || N > (nf3 ? 16 : 32)) return false;
  // NF3: both bulk copies need 16-byte multiples (N * D/64 a multiple of 8)
  if (nf3 && (D % 64 != 0 || ((int64_t)N * (D / 64)) % 8 != 0)) return false;
  const GroupLayout L = group_layout<4>(N, D, nf3);  // the widest gate area
  return L.n_slots >= 2 && smem_bytes_for<true, 32>(D) <= 227 * 1024;
}

// ---- Shares: each layer-kernel CTA's work items and tokens (once per batch) ----
// One warp per CTA b of a G-CTA layer kernel: b's item records in processing
// order (cta_item), each step's token offset and the items' tokens in order,
// so that the CTA reads all of them in one round of loads.  Runs after
// group_plan_kernel; skipped if the plan was abandoned.
constexpr int kShareWarps = 4;

__global__ void __launch_bounds__(kShareWarps * 32) group_share_kernel(const GroupWs w, int G, int scap) {
  __shared__ int soff[kShareWarps][kShareCapLimit + 1];
  __shared__ int spos[kShareWarps][kShareCapLimit];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * kShareWarps + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) w.ctl[kCtlShareGrid] = (unsigned)G;
  if (b >= G || ld_relaxed_u32(&w.ctl[kCtlAbort]) != 0xFFFFFFFFu) return;
  const int my_n = items_of((int)ld_relaxed_u32(&w.ctl[kCtlItems]), b, G);
  int* so = soff[warp];
  int* sp = spos[warp];
  auto over = [&]() {  // beyond the capacity bound (not reached: see share_cap)
    if (lane == 0) {
      w.share_n[2 * b] = -1;
      w.share_n[2 * b + 1] = -1;
    }
  };
  if (my_n > scap) return over();
  int run = 0;
  for (int k0 = 0; k0 < my_n; k0 += 32) {
    const int k = k0 + lane;
    const int4 rec = k < my_n ? w.items[cta_item(k, my_n, b, G)] : make_int4(0, 0, 0, 0);
    int inc = rec.z;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    if (k < my_n) {
      w.share_rec[(size_t)b * scap + k] = rec;
      so[k + 1] = run + inc;
      sp[k] = rec.y;
    }
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane == 0) so[0] = 0;
  __syncwarp();
  const int n_tok = run;
  if (n_tok > scap) return over();
  for (int k = lane; k <= my_n; k += 32) w.share_off[(size_t)b * (scap + 1) + k] = so[k];
  for (int i = lane; i < n_tok; i += 32) {
    int lo = 0, hi = my_n;  // the step k with so[k] <= i < so[k + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (so[mid] <= i)
        lo = mid;
      else
        hi = mid;
    }
    w.share_tok[(size_t)b * scap + i] = w.list[sp[lo] + (i - so[lo])];
  }
  if (lane == 0) {
    w.share_n[2 * b] = my_n;
    w.share_n[2 * b + 1] = n_tok;
  }
}

// ---- Offloaded table: the batch's distinct row blocks into a staging buffer ----
// The table stays in host memory (pinned and mapped into the device's address
// space) or anywhere else the device can read.  Per batch, each distinct id's
// row block crosses the link once, read by the SMs with 16-byte loads (many in
// flight per thread: the link's latency is microseconds), and lands in a
// device staging buffer at the id's dense index; the combine then reads the
// staging buffer instead of the table.

constexpr int kStageThreads = 256;
constexpr int kStageUnroll = 4;    // accesses in flight per thread
constexpr int kStageCtasPerSm = 8;

// One array of per-id row blocks (the bf16/fp32 table, or the NF3 codes or
// scales): row block of id v at src + v * row_bytes, staged to dst + u * row_bytes.
struct StagePlane {
  const uint8_t* src;
  uint8_t* dst;
  int64_t row_bytes;
  int vec;  // bytes per access (16, 8, 4 or 2), dividing row_bytes and both bases
};

// Staging buffer layout for `rows` row blocks: the table's (or the NF3
// codes') blocks, then (NF3) the scale blocks from scales_off.
struct StageLayout {
  int64_t rows, row_bytes, scale_row_bytes, scales_off, total;
};

StageLayout stage_layout(int64_t rows, int N, int D, int elem_bytes, bool nf3) {
  StageLayout L{};
  L.rows = rows;
  if (nf3) {
    const int64_t nb = (int64_t)N * (D / 64);
    L.row_bytes = nb * 24;
    L.scale_row_bytes = nb * 2;
    L.scales_off = (rows * L.row_bytes + 255) / 256 * 256;
    L.total = L.scales_off + rows * L.scale_row_bytes;
  } else {
    L.row_bytes = (int64_t)N * D * elem_bytes;
    L.total = rows * L.row_bytes;
  }
  return L;
}

template <typename Vec>
__device__ __forceinline__ void stage_plane(const StagePlane& pl, const int* __restrict__ uid_id, int64_t U,
                                            int64_t V, unsigned* err) {
  const int64_t per_row = pl.row_bytes / (int64_t)sizeof(Vec);
  const int64_t cpr = (per_row + kStageThreads - 1) / kStageThreads;  // chunks of a row block
  const int64_t tasks = U * cpr;
  // a CTA takes kStageUnroll consecutive chunks at a time: all loads first
  for (int64_t t0 = (int64_t)blockIdx.x * kStageUnroll; t0 < tasks; t0 += (int64_t)gridDim.x * kStageUnroll) {
    Vec v[kStageUnroll];
    int64_t at[kStageUnroll];
#pragma unroll
    for (int k = 0; k < kStageUnroll; ++k) {
      at[k] = -1;
      const int64_t task = t0 + k;
      if (task < tasks) {
        const int64_t u = task / cpr;
        const int64_t e = (task - u * cpr) * kStageThreads + threadIdx.x;
        const int id = uid_id[u];
        if (id < 0 || (int64_t)id >= V) {  // a grouping built with a larger vocabulary
          if (e == 0) atomicOr(err, kErrIndex);
        } else if (e < per_row) {
          v[k] = reinterpret_cast<const Vec*>(pl.src + (int64_t)id * pl.row_bytes)[e];
          at[k] = u * per_row + e;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kStageUnroll; ++k)
      if (at[k] >= 0) reinterpret_cast<Vec*>(pl.dst)[at[k]] = v[k];
  }
}

__device__ __forceinline__ void stage_any(const StagePlane& pl, const int* uid_id, int64_t U, int64_t V,
                                          unsigned* err) {
  switch (pl.vec) {
    case 16: stage_plane<uint4>(pl, uid_id, U, V, err); break;
    case 8: stage_plane<uint2>(pl, uid_id, U, V, err); break;
    case 4: stage_plane<uint32_t>(pl, uid_id, U, V, err); break;
    default: stage_plane<uint16_t>(pl, uid_id, U, V, err); break;
  }
}

__global__ void __launch_bounds__(kStageThreads) stage_rows_kernel(const GroupWs w, const StagePlane a,
                                                                   const StagePlane b, int n_planes, int64_t V,
                                                                   int64_t cap, int* n_rows, unsigned* err) {
  int64_t U = 0;
  if (ld_relaxed_u32(&w.ctl[kCtlAbort]) == 0xFFFFFFFFu) U = (int64_t)(ld_relaxed_u32(&w.ctl[kCtlTot + kAgg]) + 1u);
  if (U > cap) {  // more distinct ids than the staging buffer holds: the grouping is not this table's
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(err, kErrIndex);
    U = cap;
  }
  if (n_rows != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *n_rows = (int)U;
  stage_any(a, w.uid_id, U, V, err);
  if (n_planes > 1) stage_any(b, w.uid_id, U, V, err);
}

// The device's address of `p` (pinned host memory mapped into the device's
// address space, or memory of the current device), or nullptr.
const void* device_view(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeManaged) return a.devicePointer;
  if (a.type == cudaMemoryTypeDevice) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || a.device != dev) return nullptr;
    return a.devicePointer;
  }
  return nullptr;  // pageable host memory: not readable by the device
}

int access_bytes(int64_t row_bytes, const void* src, const void* dst) {
  const uintptr_t m = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | (uintptr_t)row_bytes;
  return (m & 15u) == 0 ? 16 : (m & 7u) == 0 ? 8 : (m & 3u) == 0 ? 4 : 2;
}

}  // namespace

size_t offload_staging_bytes(int64_t T, int64_t V, int N, int D, int elem_bytes, bool nf3) {
  return (size_t)stage_layout(std::min(T, V), N, D, elem_bytes, nf3).total;
}

mole_status offload_stage(const void* buf, size_t bytes, int64_t T, const void* table, const void* scales,
                          int64_t V, int N, int D, int elem_bytes, bool nf3, void* staging, size_t staging_bytes,
                          int* n_rows, cudaStream_t stream) {
  GroupWs w{};
  if (carve_ws(const_cast<void*>(buf), T, padded_experts(N), &w) > bytes) return MOLE_ERR_WORKSPACE;
  const StageLayout L = stage_layout(std::min(T, V), N, D, elem_bytes, nf3);
  if ((size_t)L.total > staging_bytes) return MOLE_ERR_WORKSPACE;
  const void* src = device_view(table);
  const void* ssrc = nf3 ? device_view(scales) : nullptr;
  if (src == nullptr || (nf3 && ssrc == nullptr)) return MOLE_ERR_ARG;
  uint8_t* dst = static_cast<uint8_t*>(staging);
  StagePlane a{static_cast<const uint8_t*>(src), dst, L.row_bytes, 0};
  a.vec = access_bytes(a.row_bytes, a.src, a.dst);
  StagePlane b = a;
  if (nf3) {
    b = StagePlane{static_cast<const uint8_t*>(ssrc), dst + L.scales_off, L.scale_row_bytes, 0};
    b.vec = access_bytes(b.row_bytes, b.src, b.dst);
  }
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  // enough CTAs for every chunk of the largest possible batch, at most 8 per SM
  const int64_t cpr = (L.row_bytes / a.vec + kStageThreads - 1) / kStageThreads;
  const int64_t want = (L.rows * cpr + kStageUnroll - 1) / kStageUnroll;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)kStageCtasPerSm * n_sm));
  stage_rows_kernel<<<grid, kStageThreads, 0, stream>>>(w, a, b, nf3 ? 2 : 1, V, L.rows, n_rows, err);
  return cudaGetLastError() == cudaSuccess ? MOLE_OK : MOLE_ERR_CUDA;
}

// The batch's distinct-id count into *dst (one device int32; 0 if the
// grouping was abandoned).
__global__ void distinct_count_kernel(const GroupWs w, int* dst) {
  unsigned U = 0;
  if (ld_relaxed_u32(&w.ctl[kCtlAbort]) == 0xFFFFFFFFu) U = ld_relaxed_u32(&w.ctl[kCtlTot + kAgg]) + 1u;
  *dst = (int)U;
}

mole_status token_groups_count(const void* buf, size_t bytes, int64_t T, int N, int* dst, cudaStream_t stream) {
  GroupWs w{};
  if (carve_ws(const_cast<void*>(buf), T, padded_experts(N), &w) > bytes) return MOLE_ERR_WORKSPACE;
  distinct_count_kernel<<<1, 1, 0, stream>>>(w, dst);
  return cuda_status(cudaGetLastError());
}

// Row blocks of `table` (row_bytes each, V rows) of the batch's distinct ids
// into dst at their dense indices (at most cap rows).
mole_status gather_rows_by_uid(const void* buf, size_t bytes, int64_t T, int N, const void* table, int64_t row_bytes,
                               int64_t V, void* dst, int64_t cap, cudaStream_t stream) {
  GroupWs w{};
  if (carve_ws(const_cast<void*>(buf), T, padded_experts(N), &w) > bytes) return MOLE_ERR_WORKSPACE;
  StagePlane a{static_cast<const uint8_t*>(table), static_cast<uint8_t*>(dst), row_bytes, 0};
  a.vec = access_bytes(a.row_bytes, a.src, a.dst);
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  const int64_t cpr = (row_bytes / a.vec + kStageThreads - 1) / kStageThreads;
  const int64_t want = (cap * cpr + kStageUnroll - 1) / kStageUnroll;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)kStageCtasPerSm * n_sm));
  stage_rows_kernel<<<grid, kStageThreads, 0, stream>>>(w, a, a, 1, V, cap, nullptr, err);
  return cuda_status(cudaGetLastError());
}

mole_status combine_offload(const void* buf, size_t bytes, int64_t T, const void* h, const void* Wr,
                            const void* staging, size_t staging_bytes, int64_t V, int N, int D, bool bf16_inputs,
                            bool nf3, float* out, cudaStream_t stream) {
  GroupWs w{};
  if (carve_ws(const_cast<void*>(buf), T, padded_experts(N), &w) > bytes) return MOLE_ERR_WORKSPACE;
  const int elem = bf16_inputs ? 2 : 4;
  const StageLayout L = stage_layout(std::min(T, V), N, D, elem, nf3);
  if ((size_t)L.total > staging_bytes) return MOLE_ERR_WORKSPACE;
  const uint8_t* st = static_cast<const uint8_t*>(staging);
  const uint16_t* sc = nf3 ? reinterpret_cast<const uint16_t*>(st + L.scales_off) : nullptr;
  if (bf16_inputs && grouped_applies(T, N, D, nf3) && aligned16(Wr) && aligned16(st)) {
    GArgs p{};
    p.T = T;
    p.h = static_cast<const uint16_t*>(h);
    p.Wr = static_cast<const uint16_t*>(Wr);
    p.table = reinterpret_cast<const uint16_t*>(st);
    p.codes = st;
    p.scales = sc;
    p.N = N;
    p.D = D;
    p.out = out;
    p.err = error_word();
    p.by_uid = 1;
    p.rows = L.rows;
    if (!p.err) return MOLE_ERR_CUDA;
    const mole_status s = nf3 ? layer_dispatch<true>(p, w, stream) : layer_dispatch<false>(p, w, stream);
    if (s != MOLE_ERR_UNSUPPORTED) return s;
  }
  // the ungrouped kernels, addressing the staging buffer by each token's dense index
  return combine_dispatch(w.tok_uid, T, h, Wr, st, sc, L.rows, N, D, bf16_inputs, nf3 ? 2 : (bf16_inputs ? 0 : 1),
                          out, stream);
}

size_t token_groups_bytes(int64_t T, int N) {
  if (T <= 0 || N <= 0 || N > 32) return 0;
  return carve_ws(nullptr, T, padded_experts(N), nullptr);
}

mole_status token_groups_build(const int32_t* ids, int64_t T, int64_t V, int N, void* buf, size_t bytes,
                               cudaStream_t stream) {
  if (T > kGroupedMaxT) return MOLE_ERR_UNSUPPORTED;
  GroupWs w{};
  if (carve_ws(buf, T, padded_experts(N), &w) > bytes) return MOLE_ERR_WORKSPACE;
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, group_plan_kernel, kPlanThreads, 0) != cudaSuccess ||
      occ < 1)
    return MOLE_ERR_UNSUPPORTED;
  const int64_t grid =
      std::min<int64_t>(std::min<int64_t>((T + kPlanThreads - 1) / kPlanThreads, (int64_t)occ * n_sm), kPlanMaxGrid);
  if (cudaMemsetAsync(w.key, 0xFF, w.clear_bytes, stream) != cudaSuccess) return MOLE_ERR_CUDA;
  // cooperative launch: the grid barriers need every CTA resident
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(grid, 1));
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, group_plan_kernel, ids, T, V, w, err) != cudaSuccess) return MOLE_ERR_CUDA;
  // the shares of a one-CTA-per-SM layer kernel on this device
  if (shares_apply(T, n_sm)) {
    group_share_kernel<<<(n_sm + kShareWarps - 1) / kShareWarps, kShareWarps * 32, 0, stream>>>(
        w, n_sm, (int)share_cap(T, n_sm));
    if (cudaGetLastError() != cudaSuccess) return MOLE_ERR_CUDA;
  }
  return MOLE_OK;
}

mole_status combine_groups(const void* buf, size_t bytes, int64_t T, const void* h, const void* Wr,
                           const void* table, const uint16_t* scales, bool nf3, int N, int D, float* out,
                           cudaStream_t stream) {
  GroupWs w{};
  if (carve_ws(const_cast<void*>(buf), T, padded_experts(N), &w) > bytes) return MOLE_ERR_WORKSPACE;
  if (!grouped_applies(T, N, D, nf3)) return MOLE_ERR_UNSUPPORTED;
  GArgs p{};
  p.T = T;
  p.h = static_cast<const uint16_t*>(h);
  p.Wr = static_cast<const uint16_t*>(Wr);
  p.table = static_cast<const uint16_t*>(table);
  p.codes = static_cast<const uint8_t*>(table);
  p.scales = scales;
  p.N = N;
  p.D = D;
  p.out = out;
  p.err = error_word();
  if (!p.err) return MOLE_ERR_CUDA;
  return nf3 ? layer_dispatch<true>(p, w, stream) : layer_dispatch<false>(p, w, stream);
}

mole_status combine_grouped_dispatch(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                                     const void* table, const uint16_t* scales, int64_t V, int N, int D,
                                     bool bf16_inputs, int table_kind, float* out, void* ws, size_t ws_bytes,
                                     cudaStream_t stream) {
  if (bf16_inputs && table_kind == 0 && grouped_applies(T, N, D, false) && aligned16(Wr) && aligned16(table)) {
    mole_status st = token_groups_build(ids, T, V, N, ws, ws_bytes, stream);
    if (st != MOLE_OK) return st;
    return combine_groups(ws, ws_bytes, T, h, Wr, table, nullptr, false, N, D, out, stream);
  }
  return combine_dispatch(ids, T, h, Wr, table, scales, V, N, D, bf16_inputs, table_kind, out, stream);
}

}  // namespace mole
