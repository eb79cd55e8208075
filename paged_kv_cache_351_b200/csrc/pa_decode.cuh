// Paged decode attention for sm_100a.
//
// What it computes (gitcode repo walkthrough, section 2.1 "PagedAttention":
// the query-key dot product, the softmax normalisation and the weighted sum
// of V, over K/V that the block table gathers block by block):
//   out[i, h] = sum_t softmax_t(scale * <q[i,h], K_i[t, g]>) V_i[t, g],
//   g = h / G, K_i[t] = k_cache[block_tables[i][t / 16], g, t % 16, :].
//
// Design (a B200 re-design; the pages' thread-group/warp/block kernel and its
// x-split K layout are prior art only):
//  * The work is the list of "rows" (sequence i, kv head g) — each row is
//    ceil(ctx_i / 16) pages of 16 tokens.  One warp is one worker; all
//    workers of a persistent grid (one CTA per SM) take equal, contiguous
//    ranges of the flattened page list, so every SM streams the same number
//    of bytes whatever the length mix.  A row cut by a range boundary yields
//    per-worker partial results (normalised output and log-sum-exp).  Each
//    worker publishes its share, then adds its page count to the row's
//    counter; the worker whose pages complete the row merges the shares (in
//    worker order) and writes it, then resets the counter.  No worker waits
//    for another, so nothing depends on which CTAs are resident at once,
//    and the counters are zero again when the launch ends.  Fixed-size
//    partitions (each partition its own partial, merged by a small
//    log-sum-exp kernel) and an unsplit mode are the same loop with
//    boundaries snapped to partitions or rows.
//  * Each page of a row — 16 tokens x head_size for one kv head, 4 KiB for
//    bf16/128 — is one contiguous run in the cache layout
//    [num_blocks, num_kv_heads, 16, head_size], so a worker moves it with a
//    single 1-D bulk copy (TMA engine, no tensor map, no multicast) into its
//    own shared-memory ring, completing on an mbarrier.  The worker's lane 0
//    issues the copies; the ring keeps several pages per warp in flight.
//  * The G = H / H_kv query heads that share a kv head are handled by the
//    same worker, so every K/V page is read from HBM once per group.
//  * Online softmax in fp32 with base-2 exponentials: q is pre-scaled by
//    scale * log2(e); running max, denominator and output per head are
//    rescaled when the max grows.
//  * Lane layout inside a page: a token row is LPT 16-byte vectors; lane
//    (tg, c) = (lane / LPT, lane % LPT) handles vector c of tokens
//    tg + TPI*k, k < NT.  Partial dot products are summed across the LPT
//    lanes of a token by a halving butterfly that leaves each lane one token
//    (and half the heads), then the page max is a warp reduction and the
//    probabilities go through a small shared buffer to the lanes that
//    multiply them into V.
#pragma once

#include "pa_common.cuh"

namespace pa {

constexpr int kBS = 16;        // tokens per block (block_size)
constexpr int kMaxWarps = 16;  // workers per CTA (the most any shape allows)

// Warps per CTA the register budget allows without spills: a lane of the
// scalar path keeps the query and output of G heads x EPV dims in registers
// (2 G EPV floats); at 128 or more (bf16 G = 8) only 8 warps fit.  The FP8
// path (EPV = 16) runs 16 warps up to G = 4: its G = 1 scalar path fits in
// 128 registers, and so does its tensor-core path (G >= 2), which keeps the
// query's f16 parts in shared memory and writes its results straight from
// the MMA fragments (measured on the GQA batch-256 FP8 decode: 0.169 ms with
// 12 warps, 0.161 ms with 16).  Registers are split per SM sub-partition: 13
// to 16 warps leave 128 registers per thread, 9 to 12 warps 168, 8 warps 255.
__host__ __device__ constexpr int max_warps_for(int G, int EPV) {
  return EPV == 16 ? (G >= 8 ? 8 : 16) : (2 * G * EPV >= 128 ? 8 : 12);
}

// Smallest group size whose FP8 page math runs on the tensor cores.
constexpr int kFp8MmaMinG = 2;

enum DecodeMode : int32_t { kBalanced = 0, kFixed = 1, kNoSplit = 2 };

struct DecodeArgs {
  void* out;
  const void* q;
  const void* kc;
  const void* vc;
  const int32_t* bt;
  const int32_t* ctx;
  int64_t q_sb, q_sh;  // query strides (elements)
  int64_t o_sb, o_sh;  // out strides (elements)
  int64_t bt_stride;   // block-table row stride (elements)
  int32_t B, H, Hkv, max_nb, num_blocks;
  float scale_log2;  // scale * log2(e)
  int32_t mode;
  int32_t part_pages;  // fixed mode: pages per partition
  int32_t P_max;       // fixed mode: partition capacity per (seq, head)
  int32_t stages;      // ring depth per warp
  float* ws_o;         // fixed mode: one partial output per partition (normalised)
  float* ws_lse;       // fixed mode: its log-sum-exp (natural log)
  float* sh_o;         // shares of units cut between workers: two slots per worker, [G][D] outputs
  float* sh_lse;       // and [G] log-sum-exp
  unsigned int* ws_cnt;  // per cut unit (indexed by its first worker), pages counted in so far;
                         // zero before the launch, and zero again after it
  uint64_t timeout_ns;
  const float* k_scale;  // FP8 cache: per-kv-head dequantization scales (else null)
  const float* v_scale;
  // Shared-prefix (cascade) decode: the batch is cut into groups of
  // consecutive sequences whose block tables begin with the same blocks.
  const int32_t* grp_start;   // [n_groups + 1]: group v = sequences grp_start[v] .. grp_start[v+1] - 1
  const int32_t* grp_blocks;  // [n_groups]: leading blocks every member shares
  int32_t n_groups;
  int32_t grp_members;  // most members a group may have (a group row carries members x g_real query rows)
  int32_t g_real;       // query heads per kv head
};

// Decode kinds: a plain decode, or a shared-prefix decode.  In the latter a
// row is (group, kv head) and carries the G query heads of every member of
// the group (members x g_real query rows); its pages are the group's shared
// blocks, which every member's rows attend, followed by each member's own
// remaining blocks, which only that member's rows attend (the other rows are
// masked).  A shared page is thus read once for the whole group, and each
// member's output is complete at the row's end: no second pass.
enum DecodeKind : int { kPlain = 0, kGroup = 1 };

// Tkv: cache element type (fp32, bf16 or e4m3 codes); Tq: query/output type.
template <typename Tkv, typename Tq, int D, int G>
struct DecodeCfg {
  static constexpr int ROWB = D * int(sizeof(Tkv));  // bytes of one token's K (or V) for one head
  static constexpr int LPT = ROWB / 16;              // lanes per token row
  static constexpr int TPI = 32 / LPT;               // token rows per warp-wide 16-byte load
  static constexpr int NT = kBS / TPI;               // tokens per lane per page
  static constexpr int EPV = 16 / int(sizeof(Tkv));  // cache elements per 16-byte vector (dims per lane)
  static constexpr int QROWB = D * int(sizeof(Tq));  // bytes of one query (or output) row
  static constexpr int EPQ = 16 / int(sizeof(Tq));   // query elements per 16-byte vector
  static constexpr int QV = EPV / EPQ;               // query vectors per lane per head
  static constexpr int PAGE = kBS * ROWB;            // bytes of one page
  static constexpr int QBYTES = G * QROWB;           // the group's query rows
  static constexpr int STAGE = 2 * PAGE + QBYTES;  // K page, V page, query rows
  static constexpr int GH = G >= 2 ? G / 2 : 1;    // heads a lane holds after the butterfly
  // FP8 cache, G >= kFp8MmaMinG: tensor-core page math, whose f16 query
  // parts live in shared memory after the probabilities: for G <= 4 (PACKQ)
  // a head's high and low parts are two columns of one 8-column B fragment,
  // 16 words per lane; for G = 8 both parts, 2 x 16 words for each of the
  // 4 G lanes that hold a head
  static constexpr bool MMA = sizeof(Tkv) == 1 && G >= kFp8MmaMinG;
  static constexpr bool PACKQ = MMA && G <= 4;
  static constexpr int QLO = !MMA ? 0 : PACKQ ? 32 * 64 : 4 * G * 128;
  static constexpr int PBUF = G * kBS * 4 + QLO;   // probabilities of one page (+ the query parts)
  static constexpr int LOG2_NT = NT == 16 ? 4 : NT == 8 ? 3 : NT == 4 ? 2 : NT == 2 ? 1 : 0;
  static_assert(LPT >= 8 && LPT <= 32 && (LPT & (LPT - 1)) == 0, "row of 128, 256 or 512 bytes");
  static_assert(2 * NT == LPT, "lane layout");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  static_assert(QV >= 1 && QV * EPQ == EPV, "query row split");
  // per-warp region: [ring: stages * STAGE][probabilities: PBUF][mbarriers: stages * 8], 128-byte multiple
  static constexpr size_t warp_bytes(int stages) {
    return (size_t(stages) * STAGE + PBUF + size_t(stages) * 8 + 127) / 128 * 128;
  }
};

// smem carve-up: [scan scratch: 32 int32][S: (U+1) int32][PB: X int32],
// padded to 128 bytes, then one region per warp (DecodeCfg::warp_bytes).  U
// is the number of row sequences (the batch, or the groups of a
// shared-prefix decode); X is U for a shared-prefix decode (each group's
// shared block count), else 0.
__host__ __device__ inline size_t decode_prefix_bytes(int U, int X = 0) {
  return (size_t(U + 1 + 32 + X) * 4 + 127) / 128 * 128;
}

// Groups of a shared-prefix decode must tile the batch in order
// (grp_start[0] = 0, non-decreasing, grp_start[n_groups] = B) with at most
// grp_members members each.  Block-wide check (every CTA reaches the same
// verdict); anything else sets PA_DEV_BAD_CONTEXT and the call decodes every
// sequence on its own (each its own group, nothing shared).
__device__ __forceinline__ bool groups_tile_batch(const DecodeArgs& a) {
  int ok = 1;
  const int n = a.n_groups;
  for (int v = threadIdx.x; v <= n; v += blockDim.x) {
    const int x = __ldg(a.grp_start + v);
    if (v == 0 && x != 0) ok = 0;
    if (v == n && x != a.B) ok = 0;
    if (v < n) {
      const int y = __ldg(a.grp_start + v + 1);
      if (y < x || y - x > a.grp_members) ok = 0;
    }
  }
  ok = __syncthreads_and(ok);
  if (!ok && blockIdx.x == 0 && threadIdx.x == 0) flag(PA_DEV_BAD_CONTEXT);
  return ok != 0;
}

// Shared leading blocks of group v: grp_blocks[v] (0 for a group of one),
// capped at every member's count of full blocks (a cap sets
// PA_DEV_BAD_CONTEXT).
__device__ __forceinline__ int group_prefix_blocks(const DecodeArgs& a, int v, int ctx_cap) {
  const int s0 = __ldg(a.grp_start + v), s1 = __ldg(a.grp_start + v + 1);
  int b = __ldg(a.grp_blocks + v);
  if (s1 - s0 <= 1 || b <= 0) return 0;
  for (int m = s0; m < s1; ++m) {
    const int raw = __ldg(a.ctx + m);
    const int full = (raw < 0 ? 0 : (raw > ctx_cap ? ctx_cap : raw)) / 16;
    if (b > full) {
      if (blockIdx.x == 0) flag(PA_DEV_BAD_CONTEXT);
      b = full;
    }
  }
  return b;
}

// Where page p of a group row lies: in the shared part (m = -1) or in member
// m's own pages (its table from index pb on); q = page within that part,
// e = pages of that part.  Members are walked in order, skipping those with
// no page of their own.
struct GroupCursor {
  int s0, n, pb;  // first member, members, shared blocks
  int m, q, e;
};

__device__ __forceinline__ int member_pages(const DecodeArgs& a, int seq, int pb, int ctx_cap) {
  const int raw = __ldg(a.ctx + seq);
  return ((raw < 0 ? 0 : (raw > ctx_cap ? ctx_cap : raw)) + 15) / 16 - pb;
}

__device__ __forceinline__ void group_seek(GroupCursor& g, const DecodeArgs& a, bool groups_ok, const int* PB, int v,
                                           int p, int ctx_cap) {
  g.s0 = groups_ok ? __ldg(a.grp_start + v) : v;
  g.n = groups_ok ? __ldg(a.grp_start + v + 1) - g.s0 : 1;
  g.pb = PB[v];
  if (p < g.pb) {
    g.m = -1, g.q = p, g.e = g.pb;
    return;
  }
  int q = p - g.pb;
  for (int m = 0; m < g.n; ++m) {
    const int e = member_pages(a, g.s0 + m, g.pb, ctx_cap);
    if (q < e) {
      g.m = m, g.q = q, g.e = e;
      return;
    }
    q -= e;
  }
  g.m = g.n, g.q = 0, g.e = 0;  // past the row (not reached for pages of the row)
}

__device__ __forceinline__ void group_next(GroupCursor& g, const DecodeArgs& a, int ctx_cap) {
  if (++g.q < g.e) return;
  g.q = 0;
  do {
    ++g.m;
    g.e = g.m < g.n ? member_pages(a, g.s0 + g.m, g.pb, ctx_cap) : 0;
  } while (g.e == 0 && g.m < g.n);
}

// Block-wide exclusive scan of one int per thread; returns the prefix and
// writes the total to *total.  scratch: >= 32 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    scratch[lane] = t;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int warp_prefix = warp ? scratch[warp - 1] : 0;
  *total = scratch[nw - 1];
  __syncthreads();
  return warp_prefix + x - v;
}

__device__ __forceinline__ int clamp_ctx(int c, int cap) { return c < 0 ? 0 : (c > cap ? cap : c); }

// Position of flat page index x in the row list: seq i, kv head g, page p.
struct RowPos {
  int i, g, p, np;
};

__device__ __forceinline__ RowPos locate(const int* S, int B, int Hkv, int64_t x) {
  // largest i in [0, B) with S[i] <= x (S nondecreasing, S[B] > x)
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (S[mid] <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  RowPos r;
  r.i = lo;
  r.np = (S[lo + 1] - S[lo]) / Hkv;
  const int off = int(x - S[lo]);
  r.g = off / r.np;
  r.p = off - r.g * r.np;
  return r;
}

// Snap a range boundary down to the start of its row (unsplit mode); the
// balanced and fixed modes keep page granularity.
__device__ __forceinline__ int64_t snap_boundary(const int* S, int B, int Hkv, int64_t b, int64_t W, int mode) {
  if (b >= W || mode != kNoSplit) return b < W ? b : W;
  const RowPos r = locate(S, B, Hkv, b);
  return int64_t(S[r.i]) + int64_t(r.g) * r.np;
}

// The unit a page belongs to: its row, or in fixed mode its partition of the
// row.  A unit cut by a worker boundary is merged from its pieces by the
// worker that completes it.  Returns the unit's first flat page and size.
__device__ __forceinline__ void unit_of(const RowPos& r, const int* S, int mode, int part_pages, int64_t* first,
                                        int* np) {
  const int64_t rf = int64_t(S[r.i]) + int64_t(r.g) * r.np;
  if (mode == kFixed) {
    const int u0 = (r.p / part_pages) * part_pages;
    *first = rf + u0;
    *np = min(part_pages, r.np - u0);
  } else {
    *first = rf;
    *np = r.np;
  }
}

// Writes one lane's EPV output values of a row (QV 16-byte vectors of Tq).
template <typename Tq, int EPV>
__device__ __forceinline__ void store_out(Tq* dst, const float* f) {
  constexpr int EPQ = 16 / int(sizeof(Tq));
#pragma unroll
  for (int v = 0; v < EPV / EPQ; ++v) *reinterpret_cast<uint4*>(dst + v * EPQ) = Elem<Tq>::pack(f + v * EPQ);
}

// Writes PER consecutive output values (PER = 2 or 4; 8 or 16 bytes).
template <typename Tq, int PER>
__device__ __forceinline__ void store_out_small(Tq* dst, const float* f) {
  if constexpr (sizeof(Tq) == 4) {
    if constexpr (PER == 4)
      *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
    else
      *reinterpret_cast<float2*>(dst) = make_float2(f[0], f[1]);
  } else {
    uint32_t w[PER / 2];
#pragma unroll
    for (int k = 0; k < PER / 2; ++k) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
      w[k] = *reinterpret_cast<uint32_t*>(&h);
    }
    if constexpr (PER == 4)
      *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    else
      *reinterpret_cast<uint32_t*>(dst) = w[0];
  }
}

// ---- balanced split: shares of a row cut by worker boundaries --------------
// Worker k owns the flat pages [ceil(k W / N), ceil((k+1) W / N)); page x
// belongs to worker floor(x N / W).  A cut row leaves one share per worker
// that holds some of its pages: the row's first worker wa publishes in its
// "tail" slot (2 wa + 1), every later one in its "head" slot (2 k), since a
// worker's range can begin inside one cut row and end inside another.
__device__ __forceinline__ bool worker_empty(int64_t k, int64_t W, int64_t N) {
  return (k * W + N - 1) / N == ((k + 1) * W + N - 1) / N;
}

__device__ __forceinline__ int64_t share_slot(int64_t k, int64_t wa) { return 2 * k + (k == wa ? 1 : 0); }

// Counts `mine` pages of a row into its counter (one lane; every lane of the
// warp has published its part of the share before a warp barrier).  True for
// the worker whose pages complete the row: it resets the counter, so every
// counter is zero again when the launch ends, and it alone merges the row.
// Nobody waits for anybody.  A counter that overshoots the row (a workspace
// whose counters did not start at zero) sets PA_DEV_BAD_WORKSPACE.
__device__ __forceinline__ bool count_in(unsigned int* cnt, unsigned int mine, unsigned int total) {
  // acquire-release: the caller's share (made visible to this lane by the
  // warp barrier before) is released with the count, and the last arriver
  // acquires every other worker's share with it
  unsigned int old;
  asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(cnt), "r"(mine) : "memory");
  const unsigned int now = old + mine;
  if (now < total) return false;
  // nobody else touches the counter again in this launch
  asm volatile("st.relaxed.gpu.u32 [%0], %1;" ::"l"(cnt), "r"(0u) : "memory");
  if (now > total) {
    flag(PA_DEV_BAD_WORKSPACE);
    return false;
  }
  return true;
}

// Warp-collective: publish-then-count for this warp's share of a cut row.
// Returns (in every lane) whether this worker completes the row.  The warp
// barriers order every lane's share stores before lane 0's release, and
// lane 0's acquire before every lane's reads of the other shares.
__device__ __forceinline__ bool share_done(unsigned int* cnt, int mine, int total) {
  __syncwarp();
  int last = 0;
  if ((threadIdx.x & 31) == 0) last = count_in(cnt, unsigned(mine), unsigned(total));
  last = __shfl_sync(0xffffffffu, last, 0);
  __syncwarp();
  return last != 0;
}

// Warp-collective log-sum-exp merge of the shares of one cut row (workers
// wa .. wb, in that order, so the result does not depend on which worker
// finished last).  Lane l ends with dims [l PER, l PER + PER) of each of the
// G query rows (normalised) and the rows' natural-log lse.  The shares are
// taken 32 at a time: lane t loads the lse values of share k0 + t and turns
// them into weights, which are then broadcast while every lane streams its
// dims of each share's outputs; the output loads of several shares are in
// flight at once (a long row can have tens of shares, and the merge sits at
// the end of the launch).
template <int D, int G>
__device__ __forceinline__ void merge_shares(const float* ws_o, const float* ws_lse, int64_t wa, int64_t wb,
                                             int64_t W, int64_t N, float (&acc)[G][D / 32], float (&lse)[G]) {
  constexpr int PER = D / 32;
  constexpr float kLog2e = 1.4426950408889634f;
  const int lane = threadIdx.x & 31;
  // the lse values of the first 32 shares stay in registers (lane t: share
  // wa + t); most rows have only a few shares
  float l0[G], mx[G], wsum[G];
  {
    const int64_t kl = wa + lane;
    const bool mine = kl <= wb && !worker_empty(kl, W, N);
#pragma unroll
    for (int j = 0; j < G; ++j) l0[j] = mine ? __ldcg(ws_lse + share_slot(kl, wa) * G + j) : -INFINITY;
  }
#pragma unroll
  for (int j = 0; j < G; ++j) mx[j] = l0[j];
  for (int64_t k = wa + 32 + lane; k <= wb; k += 32) {
    if (worker_empty(k, W, N)) continue;
    const int64_t slot = share_slot(k, wa);
#pragma unroll
    for (int j = 0; j < G; ++j) mx[j] = fmaxf(mx[j], __ldcg(ws_lse + slot * G + j));
  }
#pragma unroll
  for (int j = 0; j < G; ++j) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], o));
    wsum[j] = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[j][e] = 0.f;
  }
  for (int64_t k0 = wa; k0 <= wb; k0 += 32) {
    // this lane's share of the chunk: its weights (0 for none, and for a row
    // with no weight anywhere: a row of a group that attended nothing)
    const int64_t kl = k0 + lane;
    float wl[G];
    if (k0 == wa) {
#pragma unroll
      for (int j = 0; j < G; ++j) wl[j] = (l0[j] != -INFINITY && mx[j] != -INFINITY) ? ex2((l0[j] - mx[j]) * kLog2e) : 0.f;
    } else {
      const bool mine = kl <= wb && !worker_empty(kl, W, N);
#pragma unroll
      for (int j = 0; j < G; ++j)
        wl[j] = (mine && mx[j] != -INFINITY) ? ex2((__ldcg(ws_lse + share_slot(kl, wa) * G + j) - mx[j]) * kLog2e)
                                              : 0.f;
    }
    const int n = int(wb - k0 + 1 < 32 ? wb - k0 + 1 : 32);
#pragma unroll 4
    for (int t = 0; t < n; ++t) {
      float w[G];
      bool any = false;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        w[j] = __shfl_sync(0xffffffffu, wl[j], t);
        any |= w[j] != 0.f;
      }
      // a share of no weight (an empty worker's slot, never written) is skipped
      if (!any) continue;
      const int64_t slot = share_slot(k0 + t, wa);
#pragma unroll
      for (int j = 0; j < G; ++j) {
        wsum[j] += w[j];
        const float* src = ws_o + (slot * G + j) * D + lane * PER;
        float v[PER];
        if constexpr (PER == 4) {
          const float4 v4 = __ldcg(reinterpret_cast<const float4*>(src));
          v[0] = v4.x, v[1] = v4.y, v[2] = v4.z, v[3] = v4.w;
        } else {
          const float2 v2 = __ldcg(reinterpret_cast<const float2*>(src));
          v[0] = v2.x, v[1] = v2.y;
        }
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[j][e] = fmaf(w[j], v[e], acc[j][e]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const float inv = wsum[j] > 0.f ? 1.f / wsum[j] : 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[j][e] *= inv;
    lse[j] = wsum[j] > 0.f ? mx[j] + logf(wsum[j]) : -INFINITY;
  }
}

template <typename Tkv, typename Tq, int D, int G, int CK = kPlain>
__global__ void __launch_bounds__(max_warps_for(G, 16 / int(sizeof(Tkv))) * 32, 1) decode_kernel(const DecodeArgs a) {
  using C = DecodeCfg<Tkv, Tq, D, G>;
  using T = Tkv;
  constexpr int LPT = C::LPT, TPI = C::TPI, NT = C::NT, EPV = C::EPV, GH = C::GH, QV = C::QV, EPQ = C::EPQ;
  extern __shared__ __align__(128) unsigned char smem[];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int tg = lane / LPT, c = lane % LPT;
  // Row sequences: the batch's sequences, or in a shared-prefix decode its
  // groups (each sequence its own group if the groups are malformed).  The
  // shared-memory layout is sized for the larger of the two.
  const int Hkv = a.Hkv, H = a.H;
  const int ctx_cap = a.max_nb * kBS;
  const int Umax = CK == kGroup ? max(a.n_groups, a.B) : a.B;

  int* scan_scratch = reinterpret_cast<int*>(smem);
  int* S = scan_scratch + 32;
  int* PB = S + Umax + 1;  // shared-prefix decode: each group's shared blocks
  unsigned char* wbase =
      smem + decode_prefix_bytes(Umax, CK == kGroup ? Umax : 0) + size_t(warp) * C::warp_bytes(a.stages);
  unsigned char* ring = wbase;
  float* pbuf = reinterpret_cast<float*>(wbase + size_t(a.stages) * C::STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(wbase + size_t(a.stages) * C::STAGE + C::PBUF);

  if (lane == 0) {
    for (int s = 0; s < a.stages; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_barrier_init();
  }

  // Inputs may come from the kernel just before this one in the stream.
  pdl_wait();
  pdl_launch_dependents();

  // ---- prologue: page prefix over row sequences (every CTA computes it) ----
  bool groups_ok = false;
  if constexpr (CK == kGroup) groups_ok = groups_tile_batch(a);
  const int U = groups_ok ? a.n_groups : a.B;
  {
    const int nt = blockDim.x;
    const int per = (U + nt - 1) / nt;
    const int i0 = threadIdx.x * per;
    const int i1 = min(U, i0 + per);
    int local = 0;
    for (int i = i0; i < i1; ++i) {
      int np;
      if constexpr (CK == kGroup) {
        // shared blocks, then every member's own
        const int pb = groups_ok ? group_prefix_blocks(a, i, ctx_cap) : 0;
        const int s0 = groups_ok ? __ldg(a.grp_start + i) : i;
        const int n = groups_ok ? __ldg(a.grp_start + i + 1) - s0 : 1;
        PB[i] = pb;
        np = pb;
        for (int m = 0; m < n; ++m) {
          const int raw = a.ctx[s0 + m];
          if ((raw < 0 || raw > ctx_cap) && blockIdx.x == 0) flag(PA_DEV_BAD_CONTEXT);
          np += (clamp_ctx(raw, ctx_cap) + kBS - 1) / kBS - pb;
        }
      } else {
        const int raw = a.ctx[i];
        if ((raw < 0 || raw > ctx_cap) && blockIdx.x == 0) flag(PA_DEV_BAD_CONTEXT);
        np = (clamp_ctx(raw, ctx_cap) + kBS - 1) / kBS;
      }
      S[i] = np;  // this thread's own entries: pages first, prefix below
      local += np * Hkv;
    }
    int total;
    int run = block_exclusive_scan(local, scan_scratch, &total);
    for (int i = i0; i < i1; ++i) {
      const int np = S[i];
      S[i] = run;
      run += np * Hkv;
    }
    if (threadIdx.x == 0) S[U] = total;
    __syncthreads();
  }
  __syncwarp();

  const int64_t W = S[U];
  const int64_t nworkers = int64_t(gridDim.x) * nwarps;
  const int64_t wid = int64_t(blockIdx.x) * nwarps + warp;
  int64_t lo = (wid * W + nworkers - 1) / nworkers;
  int64_t hi = ((wid + 1) * W + nworkers - 1) / nworkers;
  lo = snap_boundary(S, U, Hkv, lo, W, a.mode);
  hi = snap_boundary(S, U, Hkv, hi, W, a.mode);
  const uint64_t pol = policy_evict_first();
  const Tq* qg = reinterpret_cast<const Tq*>(a.q);
  const unsigned char* kcb = reinterpret_cast<const unsigned char*>(a.kc);
  const unsigned char* vcb = reinterpret_cast<const unsigned char*>(a.vc);

  if (lo < hi) {
    // ---- producer cursor (warp-uniform) ----
    RowPos pc = locate(S, U, Hkv, lo);
    int64_t px = lo;
    int win_seq = -1, win_base = 0, win_blk = 0;  // lane-held window of 32 block ids of one table row
    int p_seg_first = 1;                          // next issued page opens a segment
    GroupCursor pg;                               // shared-prefix decode: where page pc.p lies
    if constexpr (CK == kGroup) group_seek(pg, a, groups_ok, PB, pc.i, pc.p, ctx_cap);

    auto issue = [&](int s) {
      // block id of the page (warp-collective): page pc.p of sequence pc.i,
      // or in a group row the shared page or the member's own page
      int trow = pc.i, tpage = pc.p;
      if constexpr (CK == kGroup) {
        trow = pg.m < 0 ? pg.s0 : pg.s0 + pg.m;
        tpage = pg.m < 0 ? pg.q : pg.pb + pg.q;
      }
      if (trow != win_seq || tpage < win_base || tpage >= win_base + 32) {
        win_seq = trow;
        win_base = tpage & ~31;
        const int pp = win_base + lane;
        win_blk = pp < a.max_nb ? a.bt[int64_t(trow) * a.bt_stride + pp] : 0;
      }
      int blk = __shfl_sync(0xffffffffu, win_blk, tpage - win_base);
      if (unsigned(blk) >= unsigned(a.num_blocks)) {
        if (lane == 0) flag(PA_DEV_BAD_BLOCK);
        blk = 0;
      }
      if (lane == 0) {
        const uint32_t bar = smem_u32(&bars[s]);
        unsigned char* st = ring + size_t(s) * C::STAGE;
        const int64_t page_off = (int64_t(blk) * Hkv + pc.g) * C::PAGE;
        // order this warp's earlier shared-memory reads of the stage before the async-proxy refill
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if constexpr (CK == kGroup) {
          // query rows of the group's members (rows past the last member are not loaded)
          const int nq = p_seg_first ? pg.n * a.g_real : 0;
          mbar_arrive_expect_tx(bar, 2 * C::PAGE + nq * C::QROWB);
          bulk_g2s(smem_u32(st), kcb + page_off, C::PAGE, bar, pol);
          bulk_g2s(smem_u32(st + C::PAGE), vcb + page_off, C::PAGE, bar, pol);
          for (int r = 0; r < nq; ++r)
            bulk_g2s(smem_u32(st + 2 * C::PAGE + r * C::QROWB),
                     qg + int64_t(pg.s0 + r / a.g_real) * a.q_sb + int64_t(pc.g * a.g_real + r % a.g_real) * a.q_sh,
                     C::QROWB, bar, pol);
        } else {
          mbar_arrive_expect_tx(bar, 2 * C::PAGE + (p_seg_first ? C::QBYTES : 0));
          bulk_g2s(smem_u32(st), kcb + page_off, C::PAGE, bar, pol);
          bulk_g2s(smem_u32(st + C::PAGE), vcb + page_off, C::PAGE, bar, pol);
          if (p_seg_first) {
#pragma unroll
            for (int j = 0; j < G; ++j)
              bulk_g2s(smem_u32(st + 2 * C::PAGE + j * C::QROWB),
                       qg + int64_t(pc.i) * a.q_sb + int64_t(pc.g * G + j) * a.q_sh, C::QROWB, bar, pol);
          }
        }
      }
      // advance the producer cursor
      ++px;
      ++pc.p;
      p_seg_first = 0;
      if (pc.p == pc.np) {
        pc.p = 0;
        p_seg_first = 1;
        if (++pc.g == Hkv) {
          pc.g = 0;
          do {
            ++pc.i;
          } while (pc.i < U && S[pc.i + 1] == S[pc.i]);
          if (pc.i < U) pc.np = (S[pc.i + 1] - S[pc.i]) / Hkv;
        }
        if constexpr (CK == kGroup)
          if (pc.i < U) group_seek(pg, a, groups_ok, PB, pc.i, 0, ctx_cap);
      } else {
        if constexpr (CK == kGroup) group_next(pg, a, ctx_cap);
        if (a.mode == kFixed && pc.p % a.part_pages == 0) p_seg_first = 1;
      }
    };

    const int npre = int(hi - lo < int64_t(a.stages) ? hi - lo : int64_t(a.stages));
    for (int s = 0; s < npre; ++s) issue(s);

    // ---- consumer state ----
    RowPos cc = locate(S, U, Hkv, lo);
    int64_t cx = lo;
    int seg_p0 = cc.p;
    bool seg_first = true;
    GroupCursor cg;  // shared-prefix decode: where page cc.p lies
    if constexpr (CK == kGroup) group_seek(cg, a, groups_ok, PB, cc.i, cc.p, ctx_cap);
    float q[G][EPV];
    float o[G][EPV];
    float m[G], lpart[GH];
    // FP8 cache, G >= 2: the page math runs on the tensor cores (mma.sync m16n8k16,
    // f16 operands, fp32 accumulation), lane = 4 gr + tig.  QK^T: the page's
    // 16 tokens are the M rows, the heads (padded to 8) the N columns, and
    // lane (gr, tig) feeds dims [32 tig, 32 tig + 32) of rows gr and gr + 8
    // (the contraction index is permuted the same way in both operands).
    // PV is computed as O^T = V^T P with the dims as M rows: lane (gr, tig)
    // accumulates dims [16 gr, 16 gr + 16) of heads 2 tig and 2 tig + 1.
    // Measured on B200 against the scalar path below (fp32 query): 0.274 ->
    // 0.191 ms at G = 4 (GQA batch 256); at G = 1 the scalar path is faster
    // (0.084 vs 0.089 ms on LLaMA-7B batch 64) and stays.
    // (A bf16 variant of this layout for G >= 4 — bf16 operands straight
    // from shared memory, P as bf16 high and low parts — was measured slower
    // than the CUDA-core path below: 0.241 vs 0.219 ms on the GQA batch-256
    // decode; its 16-byte operand loads hit 4x the shared-memory wavefronts
    // of the conflict-free scalar layout, since the page rows are 256 bytes
    // apart.  Not kept.)
    constexpr bool kMma = C::MMA;
    const int gr = lane >> 2, tig = lane & 3;
    // query of head gr as f16 pairs of this lane's 32 dims (qf) and the f16
    // rounding error of qf (ql; q = qf + ql to about 2^-22), kept in shared
    // memory for the lanes of real heads (lane = 4 gr + tig < 4 G; the other
    // lanes' query is zero): vector v (4 words) of lane l at qhl[v * 4 G + l],
    // qf in v = 0..3, ql in v = 4..7
    uint4* const qhl = reinterpret_cast<uint4*>(pbuf + G * kBS);
    // G <= 4: the B fragment's 8 columns are each head's high part (column
    // 2 h) and low part (column 2 h + 1), so one MMA per k-step covers both
    // and lane (gr, tig) ends with both parts of head tig's scores; lane
    // (gr, tig) keeps the part that column gr holds (head gr >> 1) at
    // qhl[v * 32 + lane], v = 0..3.  Its softmax state (mh[0], lh[0]) is then
    // that of head tig.
    float oacc[8][4];    // O^T fragments
    float mh[2], lh[2];  // running max and denominator of heads 2 tig, 2 tig + 1
    float sfac[2];       // power-of-two factor undoing the query's range normalisation
    float vscale = 1.f;
    int ctx_i = 0;
    int nreal = G;       // query rows that belong to a sequence (a group row: members x g_real)
    uint32_t phase = 0;  // bit s = parity of the next wait on stage s
    int s = 0;

    while (cx < hi) {
      unsigned char* st = ring + size_t(s) * C::STAGE;
      const uint32_t bar = smem_u32(&bars[s]);
      if (!mbar_wait_bounded(bar, (phase >> s) & 1u, a.timeout_ns)) {
        // give up: wait (bounded) for every other copy still in flight, then stop
        // (at most `stages` pages are in flight, each in its own stage)
        for (int64_t y = cx + 1; y < px; ++y) {
          const int s2 = int((s + (y - cx)) % a.stages);
          mbar_wait_bounded(smem_u32(&bars[s2]), (phase >> s2) & 1u, a.timeout_ns);
        }
        // Count the unfinished shares in (their rows are left unwritten; the
        // status word reports the timeout) so the counters end at zero.  A
        // worker holds pages of at most two cut units: one that began in an
        // earlier worker (counted in once the consumer has passed its end)
        // and one that continues in a later one (at the end of the range,
        // not yet counted in while the consumer is inside the range).
        if (lane == 0 && a.mode != kNoSplit) {
          int64_t f0, f1;
          int n0, n1;
          unit_of(locate(S, U, Hkv, lo), S, a.mode, a.part_pages, &f0, &n0);
          const int64_t e0 = hi < f0 + n0 ? hi : f0 + n0;
          if (lo != f0 && cx < e0) count_in(a.ws_cnt + f0 * nworkers / W, unsigned(e0 - lo), unsigned(n0));
          unit_of(locate(S, U, Hkv, hi - 1), S, a.mode, a.part_pages, &f1, &n1);
          if (hi != f1 + n1 && f1 >= lo) count_in(a.ws_cnt + wid, unsigned(hi - f1), unsigned(n1));
        }
        return;
      }
      phase ^= 1u << s;

      if (seg_first) {
        const uint4* qs = reinterpret_cast<const uint4*>(st + 2 * C::PAGE);
        // FP8 cache: fold the K dequantization scale into the query
        const float qscale = a.scale_log2 * (a.k_scale ? __ldg(a.k_scale + cc.g) : 1.f);
        vscale = a.v_scale ? __ldg(a.v_scale + cc.g) : 1.f;
        if constexpr (CK == kGroup) nreal = cg.n * a.g_real;
        if constexpr (kMma) {
          float qv[32];
          const int hq = C::PACKQ ? (gr >> 1) : gr;  // the head whose query this lane holds
          if (hq < nreal && hq < G) {
#pragma unroll
            for (int v = 0; v < 4; ++v) Elem<Tq>::unpack(qs[hq * (C::QROWB / 16) + tig * 4 + v], qv + 8 * v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) qv[e] = 0.f;
          }
          // Scale each head's query by a power of two so that its largest
          // value lies in [2^14, 2^15): inside the f16 range and far from
          // its subnormals; the scores are multiplied back exactly.
          float mx = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            qv[e] *= qscale;
            mx = fmaxf(mx, fabsf(qv[e]));
          }
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const int ex = mx > 0.f ? ilogbf(mx) - 14 : 0;
          const float down = ldexpf(1.f, -ex);
          uint32_t qf[16], ql[16];
#pragma unroll
          for (int j2 = 0; j2 < 16; ++j2) {
            const float a0 = qv[2 * j2] * down, a1 = qv[2 * j2 + 1] * down;
            qf[j2] = pack_f16x2(a0, a1);
            float h0, h1;
            f16x2_to_f32(qf[j2], h0, h1);
            ql[j2] = pack_f16x2(a0 - h0, a1 - h1);
          }
          if constexpr (C::PACKQ) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              qhl[v * 32 + lane] = (gr & 1) == 0 ? make_uint4(qf[4 * v], qf[4 * v + 1], qf[4 * v + 2], qf[4 * v + 3])
                                                 : make_uint4(ql[4 * v], ql[4 * v + 1], ql[4 * v + 2], ql[4 * v + 3]);
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (gr < G) {
                qhl[v * 4 * G + lane] = make_uint4(qf[4 * v], qf[4 * v + 1], qf[4 * v + 2], qf[4 * v + 3]);
                qhl[(v + 4) * 4 * G + lane] = make_uint4(ql[4 * v], ql[4 * v + 1], ql[4 * v + 2], ql[4 * v + 3]);
              }
            }
          }
          const float up = ldexpf(1.f, ex);
          sfac[0] = __shfl_sync(0xffffffffu, up, (2 * tig) * 4);
          sfac[1] = __shfl_sync(0xffffffffu, up, (2 * tig + 1) * 4);
#pragma unroll
          for (int mm = 0; mm < 8; ++mm)
#pragma unroll
            for (int k = 0; k < 4; ++k) oacc[mm][k] = 0.f;
          mh[0] = mh[1] = -INFINITY;
          lh[0] = lh[1] = 0.f;
        } else {
#pragma unroll
        for (int j = 0; j < G; ++j) {
          float f[EPV];
          if (CK != kGroup || j < nreal) {
#pragma unroll
            for (int v = 0; v < QV; ++v) Elem<Tq>::unpack(qs[j * (C::QROWB / 16) + c * QV + v], f + v * EPQ);
          } else {
#pragma unroll
            for (int e = 0; e < EPV; ++e) f[e] = 0.f;  // a row past the group's last member
          }
#pragma unroll
          for (int e = 0; e < EPV; ++e) {
            q[j][e] = f[e] * qscale;
            o[j][e] = 0.f;
          }
          m[j] = -INFINITY;
        }
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) lpart[jj] = 0.f;
        }
        // tokens of the row, consumed at its last page
        if constexpr (CK != kGroup) ctx_i = clamp_ctx(a.ctx[cc.i], ctx_cap);
        seg_p0 = cc.p;
      }
      const bool last_of_row = (cc.p == cc.np - 1);
      int valid = last_of_row ? ctx_i - cc.p * kBS : kBS;
      // group row: shared pages are full and attended by every member's rows;
      // a member's own pages only by that member's rows [alo, ahi)
      int alo = 0, ahi = G;
      if constexpr (CK == kGroup) {
        if (cg.m < 0) {
          valid = kBS;
          ahi = nreal;
        } else {
          valid = cg.q == cg.e - 1 ? clamp_ctx(a.ctx[cg.s0 + cg.m], ctx_cap) - (cg.pb + cg.q) * kBS : kBS;
          alo = cg.m * a.g_real;
          ahi = alo + a.g_real;
        }
      }

      const uint4* Ks = reinterpret_cast<const uint4*>(st);
      const uint4* Vs = reinterpret_cast<const uint4*>(st + C::PAGE);

      if constexpr (kMma) {
        const unsigned char* Kb = st;
        const unsigned char* Vb = st + C::PAGE;
        // ---- S = K q^T: rows = tokens, columns = heads ----
        // four MMA chains: high and low query parts, even and odd kk (K codes are
        // exact in f16, so both products are exact before fp32 accumulation)
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        float la[4] = {0.f, 0.f, 0.f, 0.f}, lb[4] = {0.f, 0.f, 0.f, 0.f};
        {
          const uint4 x0 = *reinterpret_cast<const uint4*>(Kb + gr * 128 + tig * 32);
          const uint4 x1 = *reinterpret_cast<const uint4*>(Kb + gr * 128 + tig * 32 + 16);
          const uint4 y0 = *reinterpret_cast<const uint4*>(Kb + (gr + 8) * 128 + tig * 32);
          const uint4 y1 = *reinterpret_cast<const uint4*>(Kb + (gr + 8) * 128 + tig * 32 + 16);
          const uint32_t r0[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          const uint32_t r1[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // word kk of a row chunk: dims 32 tig + 4 kk + {0, 1} -> k 2 tig, 2 tig + 1;
            // dims + {2, 3} -> k 2 tig + 8, 2 tig + 9
            const uint32_t af[4] = {e4m3x2_lo_to_f16x2(r0[kk]), e4m3x2_lo_to_f16x2(r1[kk]),
                                    e4m3x2_hi_to_f16x2(r0[kk]), e4m3x2_hi_to_f16x2(r1[kk])};
            if constexpr (C::PACKQ) {
              const uint4 qw = qhl[(kk >> 1) * 32 + lane];
              mma_16816_f16((kk & 1) ? sb : sa, af, (kk & 1) ? qw.z : qw.x, (kk & 1) ? qw.w : qw.y);
            } else {
              const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
              const uint4 hw = gr < G ? qhl[(kk >> 1) * 4 * G + lane] : z4;
              const uint4 lw = gr < G ? qhl[(4 + (kk >> 1)) * 4 * G + lane] : z4;
              mma_16816_f16((kk & 1) ? sb : sa, af, (kk & 1) ? hw.z : hw.x, (kk & 1) ? hw.w : hw.y);
              mma_16816_f16((kk & 1) ? lb : la, af, (kk & 1) ? lw.z : lw.x, (kk & 1) ? lw.w : lw.y);
            }
          }
          if constexpr (C::PACKQ) {
            // columns 2 tig (high part) and 2 tig + 1 (low part) of head tig
#pragma unroll
            for (int k = 0; k < 4; ++k) sa[k] += sb[k];
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) sa[k] = (sa[k] + sb[k]) + (la[k] + lb[k]);
          }
        }
        // this lane's V rows, loaded before the softmax so that their latency
        // overlaps it; tokens past the context may hold any codes (NaN would
        // survive p = 0)
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
        const uint4 va = 2 * tig < valid ? *reinterpret_cast<const uint4*>(Vb + (2 * tig) * 128 + gr * 16) : zero;
        const uint4 vb =
            2 * tig + 1 < valid ? *reinterpret_cast<const uint4*>(Vb + (2 * tig + 1) * 128 + gr * 16) : zero;
        const uint4 vc =
            2 * tig + 8 < valid ? *reinterpret_cast<const uint4*>(Vb + (2 * tig + 8) * 128 + gr * 16) : zero;
        const uint4 vd =
            2 * tig + 9 < valid ? *reinterpret_cast<const uint4*>(Vb + (2 * tig + 9) * 128 + gr * 16) : zero;
        if constexpr (C::PACKQ) {
          // head tig at tokens gr and gr + 8 (log2 units)
          float t0 = (sa[0] + sa[1]) * sfac[0], t1 = (sa[2] + sa[3]) * sfac[0];
          if (gr >= valid) t0 = -INFINITY;
          if (gr + 8 >= valid) t1 = -INFINITY;
          if constexpr (CK == kGroup) {  // a row (head) that does not attend this page
            if (tig < alo || tig >= ahi) t0 = t1 = -INFINITY;
          }
          float pm = fmaxf(t0, t1);
#pragma unroll
          for (int msk = 4; msk < 32; msk <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, msk));
          const float mn = fmaxf(mh[0], pm);
          float al = ex2(mh[0] - mn);
          const bool grew = __any_sync(0xffffffffu, mn != mh[0]);
          mh[0] = mn;
          float p0 = ex2(t0 - mn), p1 = ex2(t1 - mn);
          if constexpr (CK == kGroup) {
            if (mn == -INFINITY) al = 1.f, p0 = p1 = 0.f;
          }
          lh[0] = lh[0] * al + (p0 + p1);
          if (grew) {
            // the O^T columns of this lane are heads 2 tig and 2 tig + 1: their
            // factors from lanes tig' = 2 tig, 2 tig + 1 (columns past the heads
            // hold zeros)
            const float alA = __shfl_sync(0xffffffffu, al, (2 * tig) & 3);
            const float alB = __shfl_sync(0xffffffffu, al, (2 * tig + 1) & 3);
#pragma unroll
            for (int mm = 0; mm < 8; ++mm) {
              oacc[mm][0] *= alA;
              oacc[mm][1] *= alB;
              oacc[mm][2] *= alA;
              oacc[mm][3] *= alB;
            }
          }
          // probabilities [head][token] through shared memory into the B layout of P V
          if (tig < G) {
            pbuf[tig * kBS + gr] = p0;
            pbuf[tig * kBS + gr + 8] = p1;
          }
        } else {
          // sa = {S[gr][2tig], S[gr][2tig+1], S[gr+8][2tig], S[gr+8][2tig+1]} (log2 units)
          float sc4[4] = {sa[0] * sfac[0], sa[1] * sfac[1], sa[2] * sfac[0], sa[3] * sfac[1]};
          if (gr >= valid) sc4[0] = sc4[1] = -INFINITY;
          if (gr + 8 >= valid) sc4[2] = sc4[3] = -INFINITY;
          if constexpr (CK == kGroup) {  // rows (heads) that do not attend this page
            if (2 * tig < alo || 2 * tig >= ahi) sc4[0] = sc4[2] = -INFINITY;
            if (2 * tig + 1 < alo || 2 * tig + 1 >= ahi) sc4[1] = sc4[3] = -INFINITY;
          }
          float pm0 = fmaxf(sc4[0], sc4[2]), pm1 = fmaxf(sc4[1], sc4[3]);
#pragma unroll
          for (int msk = 4; msk < 32; msk <<= 1) {
            pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, msk));
            pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, msk));
          }
          // token 0 of every page is valid, so the maxima are finite; in a
          // group row a row that has attended nothing yet keeps -inf (no
          // rescale, zero probabilities)
          const float mn0 = fmaxf(mh[0], pm0), mn1 = fmaxf(mh[1], pm1);
          float al0 = ex2(mh[0] - mn0), al1 = ex2(mh[1] - mn1);
          const bool grew = __any_sync(0xffffffffu, mn0 != mh[0] || mn1 != mh[1]);
          mh[0] = mn0;
          mh[1] = mn1;
          float p0 = ex2(sc4[0] - mn0), p1 = ex2(sc4[1] - mn1), p2 = ex2(sc4[2] - mn0), p3 = ex2(sc4[3] - mn1);
          if constexpr (CK == kGroup) {
            if (mn0 == -INFINITY) al0 = 1.f, p0 = p2 = 0.f;
            if (mn1 == -INFINITY) al1 = 1.f, p1 = p3 = 0.f;
          }
          lh[0] = lh[0] * al0 + (p0 + p2);
          lh[1] = lh[1] * al1 + (p1 + p3);
          if (grew) {
#pragma unroll
            for (int mm = 0; mm < 8; ++mm) {
              oacc[mm][0] *= al0;
              oacc[mm][1] *= al1;
              oacc[mm][2] *= al0;
              oacc[mm][3] *= al1;
            }
          }
          // probabilities [head][token] through shared memory into the B layout of P V
          if (2 * tig < G) {
            pbuf[(2 * tig) * kBS + gr] = p0;
            pbuf[(2 * tig) * kBS + gr + 8] = p2;
          }
          if (2 * tig + 1 < G) {
            pbuf[(2 * tig + 1) * kBS + gr] = p1;
            pbuf[(2 * tig + 1) * kBS + gr + 8] = p3;
          }
        }
        __syncwarp();
        uint32_t pb0 = 0u, pb1 = 0u;
        if (gr < G) {
          const float2 u = *reinterpret_cast<const float2*>(pbuf + gr * kBS + 2 * tig);
          const float2 w = *reinterpret_cast<const float2*>(pbuf + gr * kBS + 2 * tig + 8);
          pb0 = pack_f16x2(u.x, u.y);
          pb1 = pack_f16x2(w.x, w.y);
        }
        // ---- O^T += V^T P: rows = dims 16 gr + 2 mm (+1), k = tokens ----
        {
          const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
          const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            // word w: dims 16 gr + 4 w + 0..3; interleave two tokens' codes per dim
            const uint32_t lo01 = __byte_perm(wa[w], wb[w], 0x5140), hi01 = __byte_perm(wa[w], wb[w], 0x7362);
            const uint32_t lo89 = __byte_perm(wc[w], wd[w], 0x5140), hi89 = __byte_perm(wc[w], wd[w], 0x7362);
            const uint32_t f0[4] = {e4m3x2_lo_to_f16x2(lo01), e4m3x2_hi_to_f16x2(lo01), e4m3x2_lo_to_f16x2(lo89),
                                    e4m3x2_hi_to_f16x2(lo89)};
            mma_16816_f16(oacc[2 * w], f0, pb0, pb1);
            const uint32_t f1[4] = {e4m3x2_lo_to_f16x2(hi01), e4m3x2_hi_to_f16x2(hi01), e4m3x2_lo_to_f16x2(hi89),
                                    e4m3x2_hi_to_f16x2(hi89)};
            mma_16816_f16(oacc[2 * w + 1], f1, pb0, pb1);
          }
        }
      } else {
      // ---- scores: partial dot products, then the halving butterfly ----
      float acc[G][NT];
#pragma unroll
      for (int k = 0; k < NT; ++k) {
        float kf[EPV];
        Elem<T>::unpack(Ks[(tg + TPI * k) * LPT + c], kf);
#pragma unroll
        for (int j = 0; j < G; ++j) {
          // two interleaved partial sums on the packed-FMA pipe
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int e = 0; e < EPV; e += 2) ffma2(s0, s1, q[j][e], q[j][e + 1], kf[e], kf[e + 1]);
          acc[j][k] = s0 + s1;
        }
      }
#pragma unroll
      for (int step = 0; step < C::LOG2_NT; ++step) {
        const int half = (NT >> step) / 2;
        const int mask = LPT >> (step + 1);
        const bool upper = (c & mask) != 0;
#pragma unroll
        for (int j = 0; j < G; ++j) {
#pragma unroll
          for (int k = 0; k < half; ++k) {
            const float send = upper ? acc[j][k] : acc[j][k + half];
            const float keep = upper ? acc[j][k + half] : acc[j][k];
            acc[j][k] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
          }
        }
      }
      const bool hi_half = (c & 1) != 0;
      float sc[GH];
      if constexpr (G >= 2) {
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          const float send = hi_half ? acc[jj][0] : acc[jj + GH][0];
          const float keep = hi_half ? acc[jj + GH][0] : acc[jj][0];
          sc[jj] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
        }
      } else {
        sc[0] = acc[0][0] + __shfl_xor_sync(0xffffffffu, acc[0][0], 1);
      }
      const int t_own = tg + TPI * (c >> 1);
      if (t_own >= valid) {
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) sc[jj] = -INFINITY;
      }
      if constexpr (CK == kGroup) {  // rows (heads) that do not attend this page
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          const int j = (G >= 2 && hi_half) ? jj + GH : jj;
          if (j < alo || j >= ahi) sc[jj] = -INFINITY;
        }
      }

      // ---- page max, new running max, rescale factors ----
      float pm[GH];
#pragma unroll
      for (int jj = 0; jj < GH; ++jj) {
        float x = sc[jj];
#pragma unroll
        for (int msk = 2; msk < 32; msk <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, msk));
        pm[jj] = x;
      }
      float pmall[G];
      if constexpr (G >= 2) {
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          const float other = __shfl_xor_sync(0xffffffffu, pm[jj], 1);
          pmall[jj] = hi_half ? other : pm[jj];
          pmall[jj + GH] = hi_half ? pm[jj] : other;
        }
      } else {
        pmall[0] = pm[0];
      }
      float alpha[G];
      bool grew = false;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float mn = fmaxf(m[j], pmall[j]);
        alpha[j] = (CK == kGroup && mn == -INFINITY) ? 1.f : ex2(m[j] - mn);  // a row that attended nothing yet
        grew |= (mn != m[j]);
        m[j] = mn;
      }

      // ---- probabilities of this lane's (token, heads); denominators ----
#pragma unroll
      for (int jj = 0; jj < GH; ++jj) {
        const float mj = (G >= 2 && hi_half) ? m[(jj + GH) % G] : m[jj];
        const float aj = (G >= 2 && hi_half) ? alpha[(jj + GH) % G] : alpha[jj];
        const float p = (CK == kGroup && mj == -INFINITY) ? 0.f : ex2(sc[jj] - mj);
        const bool own = (G >= 2) || !hi_half;
        lpart[jj] = lpart[jj] * aj + (own ? p : 0.f);
        if (own) {
          const int j = (G >= 2 && hi_half) ? jj + GH : jj;
          pbuf[(tg * NT + (c >> 1)) * G + j] = p;
        }
      }
      __syncwarp();
      if (grew) {
#pragma unroll
        for (int j = 0; j < G; ++j)
#pragma unroll
          for (int e = 0; e < EPV; ++e) o[j][e] *= alpha[j];
      }

      // ---- weighted sum of V (probabilities read per token, heads contiguous) ----
#pragma unroll
      for (int k = 0; k < NT; ++k) {
        float pk[G];
        {
          const float* src = pbuf + (tg * NT + k) * G;
          if constexpr (G % 4 == 0) {
#pragma unroll
            for (int j4 = 0; j4 < G; j4 += 4) {
              const float4 v4 = *reinterpret_cast<const float4*>(src + j4);
              pk[j4] = v4.x, pk[j4 + 1] = v4.y, pk[j4 + 2] = v4.z, pk[j4 + 3] = v4.w;
            }
          } else if constexpr (G == 2) {
            const float2 v2 = *reinterpret_cast<const float2*>(src);
            pk[0] = v2.x, pk[1] = v2.y;
          } else {
            pk[0] = src[0];
          }
        }
        float vf[EPV];
        Elem<T>::unpack(Vs[(tg + TPI * k) * LPT + c], vf);
        if (tg + TPI * k >= valid) {
#pragma unroll
          for (int e = 0; e < EPV; ++e) vf[e] = 0.f;  // unused slots may hold any bits
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
#pragma unroll
          for (int e = 0; e < EPV; e += 2) ffma2(o[j][e], o[j][e + 1], pk[j], pk[j], vf[e], vf[e + 1]);
        }
      }
      }
      __syncwarp();  // every lane is done with stage s and with pbuf

      // ---- refill stage s with the next page of this worker's range ----
      if (px < hi) issue(s);

      // ---- segment end: combine lanes and write ----
      const bool seg_last = (cx == hi - 1) || last_of_row || (a.mode == kFixed && (cc.p + 1) % a.part_pages == 0);
      if (seg_last) {
        // Each lane owns some (query row j, chunk of EPV dims) pieces of the
        // segment's result and calls put(j, chunk, values, max, denominator,
        // writes_lse) for each.  Scalar path: lanes 0..LPT-1 (tg = 0) own
        // chunk c of every row, lane 0 writes the rows' lse.  Tensor-core
        // path: lane (gr, tig) already holds dims [16 gr, 16 gr + 16) of rows
        // 2 tig and 2 tig + 1 in its O^T fragments and writes them from
        // there (no gather into a per-lane copy of every row).
        float lall[G];
        float lrow[2];
        float mrow[2];
        if constexpr (kMma) {
          lrow[0] = lh[0];
          lrow[1] = lh[1];
#pragma unroll
          for (int msk = 4; msk < 32; msk <<= 1) {
            lrow[0] += __shfl_xor_sync(0xffffffffu, lrow[0], msk);
            lrow[1] += __shfl_xor_sync(0xffffffffu, lrow[1], msk);
          }
          mrow[0] = mh[0];
          mrow[1] = mh[1];
          if constexpr (C::PACKQ) {
            // this lane's state is head tig's; its output columns are heads
            // 2 tig and 2 tig + 1
            const float l0 = lrow[0], m0 = mh[0];
            lrow[0] = __shfl_sync(0xffffffffu, l0, (2 * tig) & 3);
            lrow[1] = __shfl_sync(0xffffffffu, l0, (2 * tig + 1) & 3);
            mrow[0] = __shfl_sync(0xffffffffu, m0, (2 * tig) & 3);
            mrow[1] = __shfl_sync(0xffffffffu, m0, (2 * tig + 1) & 3);
          }
        } else {
#pragma unroll
        for (int msk = LPT; msk < 32; msk <<= 1)
#pragma unroll
          for (int j = 0; j < G; ++j)
#pragma unroll
            for (int e = 0; e < EPV; ++e) o[j][e] += __shfl_xor_sync(0xffffffffu, o[j][e], msk);
        const bool hi_half = (c & 1) != 0;
#pragma unroll
        for (int jj = 0; jj < GH; ++jj) {
          float x = lpart[jj];
#pragma unroll
          for (int msk = 2; msk < 32; msk <<= 1) x += __shfl_xor_sync(0xffffffffu, x, msk);
          if constexpr (G >= 2) {
            const float other = __shfl_xor_sync(0xffffffffu, x, 1);
            lall[jj] = hi_half ? other : x;
            lall[jj + GH] = hi_half ? x : other;
          } else {
            lall[0] = x + __shfl_xor_sync(0xffffffffu, x, 1);
          }
        }
        }
        auto for_owned = [&](auto&& put) {
          if constexpr (kMma) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int j = 2 * tig + hh;
              if (j < G) {
                float f[EPV];
#pragma unroll
                for (int e = 0; e < EPV; ++e) f[e] = oacc[e >> 1][hh + 2 * (e & 1)];
                put(j, gr, f, mrow[hh], lrow[hh], gr == 0);
              }
            }
          } else {
            if (tg == 0) {
#pragma unroll
              for (int j = 0; j < G; ++j) put(j, c, o[j], m[j], lall[j], c == 0);
            }
          }
        };
        // This segment's unit: the row, or in fixed mode its partition.  A
        // unit that spans the whole row gives the row's output; a partition
        // of a longer row gives a partial for the merge kernel.
        const int up0 = a.mode == kFixed ? (cc.p / a.part_pages) * a.part_pages : 0;
        const int unp = a.mode == kFixed ? min(a.part_pages, cc.np - up0) : cc.np;
        const bool row_unit = unp == cc.np;
        const bool whole_unit = seg_p0 == up0 && cc.p == up0 + unp - 1;
        if (whole_unit && row_unit) {
          for_owned([&](int j, int ch, const float* f, float, float l, bool) {
            // query row j -> (sequence, head); a group row's rows past its
            // last member are dropped, and a member that attended nothing
            // (no context) gets a zero row
            int seq = cc.i, head = cc.g * G + j;
            if constexpr (CK == kGroup) {
              if (j >= nreal) return;
              seq = cg.s0 + j / a.g_real;
              head = cc.g * a.g_real + j % a.g_real;
            }
            const float inv = (CK != kGroup || l > 0.f) ? vscale / l : 0.f;
            float y[EPV];
#pragma unroll
            for (int e = 0; e < EPV; ++e) y[e] = f[e] * inv;
            store_out<Tq, EPV>(reinterpret_cast<Tq*>(a.out) + int64_t(seq) * a.o_sb + int64_t(head) * a.o_sh + ch * EPV,
                               y);
          });
        } else if (whole_unit) {
          // fixed mode: one partial per partition; a separate kernel merges them
          const int64_t base = (int64_t(cc.i) * H + int64_t(cc.g) * G) * a.P_max + cc.p / a.part_pages;
          for_owned([&](int j, int ch, const float* f, float mj, float l, bool lse_lane) {
            const float inv = vscale / l;
            float4* dst = reinterpret_cast<float4*>(a.ws_o + (base + j * a.P_max) * D + ch * EPV);
#pragma unroll
            for (int e4 = 0; e4 < EPV / 4; ++e4)
              dst[e4] = make_float4(f[4 * e4] * inv, f[4 * e4 + 1] * inv, f[4 * e4 + 2] * inv, f[4 * e4 + 3] * inv);
            if (lse_lane) a.ws_lse[base + j * a.P_max] = (mj + log2f(l)) * 0.69314718055994530942f;
          });
        } else {
          // A unit cut by a worker boundary: publish this worker's share
          // (normalised output + log-sum-exp) in its slot, then count its
          // pages in.  The worker whose pages complete the unit merges all
          // shares in worker order and writes the row (or the partition's
          // partial).
          const int64_t unit_first = int64_t(S[cc.i]) + int64_t(cc.g) * cc.np + up0;
          const int64_t wa = unit_first * nworkers / W;
          const bool is_tail = (seg_p0 == up0);
          const int64_t slot = 2 * wid + (is_tail ? 1 : 0);
          for_owned([&](int j, int ch, const float* f, float mj, float l, bool lse_lane) {
            // (a group row's row that attended nothing in this segment: a
            // zero share of weight 0)
            const float inv = (CK != kGroup || l > 0.f) ? vscale / l : 0.f;
            float4* dst = reinterpret_cast<float4*>(a.sh_o + (slot * G + j) * D + ch * EPV);
#pragma unroll
            for (int e4 = 0; e4 < EPV / 4; ++e4)
              dst[e4] = make_float4(f[4 * e4] * inv, f[4 * e4 + 1] * inv, f[4 * e4 + 2] * inv, f[4 * e4 + 3] * inv);
            if (lse_lane)
              a.sh_lse[slot * G + j] =
                  (CK == kGroup && !(l > 0.f)) ? -INFINITY : (mj + log2f(l)) * 0.69314718055994530942f;
          });
          const bool last = share_done(a.ws_cnt + wa, cc.p - seg_p0 + 1, unp);
          if (last) {
            constexpr int PER = D / 32;
            const int64_t wb = (unit_first + unp - 1) * nworkers / W;
            float acc[G][PER], lse_m[G];
            merge_shares<D, G>(a.sh_o, a.sh_lse, wa, wb, W, nworkers, acc, lse_m);
            if (!row_unit) {
              // the partition's partial, as if one worker had reduced it
              const int64_t base = (int64_t(cc.i) * H + int64_t(cc.g) * G) * a.P_max + up0 / a.part_pages;
#pragma unroll
              for (int j = 0; j < G; ++j) {
                float* dst = a.ws_o + (base + j * a.P_max) * D + lane * PER;
#pragma unroll
                for (int e = 0; e < PER; ++e) dst[e] = acc[j][e];
                if (lane == 0) a.ws_lse[base + j * a.P_max] = lse_m[j];
              }
            } else {
#pragma unroll
              for (int j = 0; j < G; ++j) {
                int seq = cc.i, head = cc.g * G + j;
                if constexpr (CK == kGroup) {
                  if (j >= nreal) continue;
                  seq = cg.s0 + j / a.g_real;
                  head = cc.g * a.g_real + j % a.g_real;
                }
                store_out_small<Tq, PER>(
                    reinterpret_cast<Tq*>(a.out) + int64_t(seq) * a.o_sb + int64_t(head) * a.o_sh + lane * PER, acc[j]);
              }
            }
          }
        }
      }

      // ---- advance the consumer cursor ----
      ++cx;
      seg_first = seg_last;
      if (++cc.p == cc.np) {
        cc.p = 0;
        if (++cc.g == Hkv) {
          cc.g = 0;
          do {
            ++cc.i;
          } while (cc.i < U && S[cc.i + 1] == S[cc.i]);
          if (cc.i < U) cc.np = (S[cc.i + 1] - S[cc.i]) / Hkv;
        }
        if constexpr (CK == kGroup)
          if (cc.i < U) group_seek(cg, a, groups_ok, PB, cc.i, 0, ctx_cap);
      } else {
        if constexpr (CK == kGroup) group_next(cg, a, ctx_cap);
      }
      if (++s == a.stages) s = 0;
    }
  }

  // ---- row sequences with no pages: zero output rows (no context; in a
  // shared-prefix decode, every member of such a group) ----
  for (int64_t i = wid; i < U; i += nworkers) {
    if (S[i + 1] != S[i]) continue;
    int s0 = int(i), n = 1;
    if constexpr (CK == kGroup) {
      if (groups_ok) {
        s0 = __ldg(a.grp_start + i);
        n = __ldg(a.grp_start + i + 1) - s0;
      }
    }
    constexpr int OVR = C::QROWB / 16;  // 16-byte vectors per output row
    for (int mm = 0; mm < n; ++mm) {
      Tq* ob = reinterpret_cast<Tq*>(a.out) + int64_t(s0 + mm) * a.o_sb;
      for (int idx = lane; idx < H * OVR; idx += 32) {
        const int h = idx / OVR, cc2 = idx % OVR;
        *reinterpret_cast<uint4*>(ob + int64_t(h) * a.o_sh + cc2 * EPQ) = make_uint4(0, 0, 0, 0);
      }
    }
  }
}

// ---- log-sum-exp merge of partial results ----------------------------------
// out = sum_p exp(lse_p - LSE) o_p, LSE = log sum_p exp(lse_p), with o_p the
// normalised partial outputs of fixed partitions.  One CTA of kMergeWarps
// warps per (sequence, query head) with more than one partition (the merge
// is bound by load latency, so many warps each keep loads in flight): warp w
// takes partitions w, w + kMergeWarps, ...; lanes first find the warp's
// largest lse, then weight 32 partitions at a time and broadcast the
// weights while every lane streams its dims (several partitions' loads in
// flight); the warps' results are combined through shared memory in warp
// order (a fixed order, so the result does not depend on timing).
constexpr int kMergeWarps = 16;

template <typename T, int D>
__global__ void __launch_bounds__(kMergeWarps * 32) merge_fixed_kernel(const DecodeArgs a, int part_tokens) {
  pdl_wait();
  constexpr int PER = D / 32;
  constexpr int NW = kMergeWarps;
  constexpr float kLog2e = 1.4426950408889634f;
  __shared__ float sm_m[NW], sm_w[NW];
  __shared__ __align__(16) float sm_acc[NW][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = blockIdx.x;  // (sequence, query head)
  if (row >= int64_t(a.B) * a.H) return;
  const int i = int(row / a.H), h = int(row % a.H);
  const int ctx = clamp_ctx(a.ctx[i], a.max_nb * kBS);
  const int np = (ctx + part_tokens - 1) / part_tokens;
  if (np <= 1) return;  // the decode kernel wrote this row itself
  const float* lse = a.ws_lse + row * a.P_max;
  const float* ob = a.ws_o + row * a.P_max * D;
  const int mine = np > warp ? (np - warp + NW - 1) / NW : 0;  // partitions of this warp
  float mw = -INFINITY;
  for (int t = lane; t < mine; t += 32) mw = fmaxf(mw, __ldcg(lse + warp + NW * t));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
  float acc[PER], wsum = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int c0 = 0; c0 < mine; c0 += 32) {
    const int tl = c0 + lane;
    const float wl = tl < mine ? ex2((__ldcg(lse + warp + NW * tl) - mw) * kLog2e) : 0.f;
    const int n = mine - c0 < 32 ? mine - c0 : 32;
#pragma unroll 8
    for (int t = 0; t < n; ++t) {
      const float w = __shfl_sync(0xffffffffu, wl, t);
      const float* src = ob + int64_t(warp + NW * (c0 + t)) * D + lane * PER;
      float v[PER];
      if constexpr (PER == 4) {
        const float4 v4 = __ldcg(reinterpret_cast<const float4*>(src));
        v[0] = v4.x, v[1] = v4.y, v[2] = v4.z, v[3] = v4.w;
      } else {
        const float2 v2 = __ldcg(reinterpret_cast<const float2*>(src));
        v[0] = v2.x, v[1] = v2.y;
      }
      wsum += w;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, v[e], acc[e]);
    }
  }
  if (lane == 0) {
    sm_m[warp] = mw;
    sm_w[warp] = wsum;
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) sm_acc[warp][lane * PER + e] = acc[e];
  __syncthreads();
  if (warp != 0) return;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < NW; ++w)
    if (sm_w[w] > 0.f) M = fmaxf(M, sm_m[w]);
  float tot = 0.f, f[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) f[e] = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    if (!(sm_w[w] > 0.f)) continue;
    const float sc = ex2((sm_m[w] - M) * kLog2e);
    tot += sc * sm_w[w];
#pragma unroll
    for (int e = 0; e < PER; ++e) f[e] = fmaf(sc, sm_acc[w][lane * PER + e], f[e]);
  }
  const float inv = 1.f / tot;
#pragma unroll
  for (int e = 0; e < PER; ++e) f[e] *= inv;
  T* dst = reinterpret_cast<T*>(a.out) + int64_t(i) * a.o_sb + int64_t(h) * a.o_sh + lane * PER;
  store_out_small<T, PER>(dst, f);
}

}  // namespace pa
