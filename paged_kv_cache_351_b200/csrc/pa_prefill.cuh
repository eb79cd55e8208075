// Multi-token (chunked-prefill) paged attention on the tensor cores (sm_100a).
//
// What it computes (gitcode repo walkthrough, section 2.2: a long prompt's
// prefill is cut into chunks that run in the same step as decode requests;
// section 2.1: the attention itself is the QK dot product, softmax and
// weighted sum of V over K/V gathered through the block table): sequence i
// brings n_i new tokens at positions c_i .. c_i + n_i - 1 (c_i = ctx_i - n_i,
// their K/V already in the cache); the query row of position p and head h
// attends keys 0 .. p of kv head h / G.
//
// Design.  One CTA owns 256 query rows of one (sequence, kv head), as two
// 128-row halves A and B: 256 / G consecutive new tokens times the G query
// heads of the kv head.  Keys stream in tiles of 128 tokens (8 pages), and
// each K/V tile in shared memory serves both halves: the bytes streamed per
// FLOP, which bound a one-half design (a K/V tile per 128 rows), are halved.
// Per tile j and half X:
//   S_X = Q_X K^T      tcgen05.mma, M = 128, N = 128, K = 128, fp32 in TMEM;
//   P_X = exp(S_X - m) 4 softmax warps per half, one query row per thread;
//   O_X += P_X V       tcgen05.mma with P_X read from TMEM (bf16 pairs that
//                      overwrite the first 64 columns of S_X), O_X in TMEM.
// TMEM holds S_A, S_B, O_A and O_B (512 columns).  The MMA order
//   PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1), PV_A(j+1), ...
// lets each half's softmax run while the tensor core works for the other.
// Q, K and V reach shared memory through tiled TMA loads with 128-byte
// swizzle: Q_X as a [128/G tokens][G heads][64 dims] box per half of the
// head dimension; each K/V page (one (block, kv head) of the cache, id from
// the block table) as a [16 tokens][64 dims] box per half.  K has three
// stages, released when QK^T of both halves is done; V has two, released
// after both PVs.  Warp roles: warp 0 issues the Q and K loads, warp 2 the V
// loads, warp 1 owns TMEM and issues the MMAs (one thread), warps 4-7 run
// the softmax and epilogue of half A and warps 8-11 those of half B.  Every
// wait is bounded by the caller's timeout (PA_DEV_TIMEOUT), after which each
// role stops, waits (bounded) for its own copies and MMAs in flight, and
// TMEM is released.
#pragma once

#include "pa_common.cuh"
#include "pa_tc.cuh"

namespace pa {

struct PrefillArgs {
  __nv_bfloat16* out;  // [T, H, 128]
  int64_t o_st, o_sh;  // element strides of out (token, head)
  const int32_t* bt;   // block tables [B, max_nb]
  int64_t bt_stride;
  const int32_t* ctx;          // [B] tokens in the cache after the step
  const int32_t* query_start;  // [B + 1] first query row of each sequence
  int32_t B, T, max_nb, num_blocks;
  float scale_log2;  // scale * log2(e), > 0
  uint64_t timeout_ns;
};

constexpr int kPfThreads = 384;      // warps 0-3: loads and MMA; 4-7: half A; 8-11: half B
constexpr int kPfRows = 256;         // query rows per CTA
constexpr uint32_t kPfHalf = 16384;  // 128 rows x 128 bytes: one 64-dim half of a 128 x 128 bf16 tile
constexpr uint32_t kPfTile = 2 * kPfHalf;
constexpr int kKStages = 3;  // K is free again once QK^T of its tile is done for both halves
constexpr int kVStages = 2;  // V is free again once PV of its tile is done for both halves
constexpr uint32_t kSmQ = 0;  // Q_A, Q_B
constexpr uint32_t kSmK = kSmQ + 2 * kPfTile;
constexpr uint32_t kSmV = kSmK + kKStages * kPfTile;
constexpr uint32_t kSmBar = kSmV + kVStages * kPfTile;
constexpr uint32_t kPfSmemBytes = kSmBar + 160 + 1024;  // + barriers + alignment slack (<= 227 KiB)
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
constexpr uint32_t kPfTmemCols = 512;
constexpr uint32_t kTmO = 256;

// Barrier slots (8 bytes each) after kSmBar.
enum PfBar : int {
  kBarQ = 0,
  kBarKFull = 1,   // + K stage (3)
  kBarKFree = 4,   // + K stage (3)
  kBarVFull = 7,   // + V stage (2)
  kBarVFree = 9,   // + V stage (2)
  kBarSFull = 11,  // + half (2)
  kBarPFull = 13,  // + half (2), 128 arrivals
  kBarODone = 15,  // + half (2)
  kBarDrain = 17,
  kBarTmemSlot = 18,  // 4-byte TMEM base address
};
static_assert(8 * kBarTmemSlot + 4 <= 160, "barrier area");
static_assert(kPfSmemBytes <= 232448, "shared memory per block");

// All lanes wait; the warp agrees on the outcome so that warp-collective
// tcgen05 instructions stay converged.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

template <int G>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
  constexpr int TOK = 128 / G;  // new tokens per half
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + kSmBar + 8u * uint32_t(i); };

  pdl_wait();
  pdl_launch_dependents();

  const int seq = blockIdx.z;
  const int kvh = blockIdx.y;
  const int qt = int(gridDim.x) - 1 - int(blockIdx.x);  // longest key ranges first
  const int q0 = a.query_start[seq];
  const int qlen = a.query_start[seq + 1] - q0;
  const int ctx = a.ctx[seq];
  if (q0 < 0 || qlen < 0 || q0 + qlen > a.T || qlen > ctx || ctx > a.max_nb * 16 ||
      qlen > int(gridDim.x) * 2 * TOK) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0) flag(PA_DEV_BAD_CONTEXT);
    return;
  }
  const int tok0 = qt * 2 * TOK;  // first new token of the CTA
  if (tok0 >= qlen) return;       // this tile holds no new token of the sequence
  const int c0 = ctx - qlen;
  const int kv_len = c0 + min(qlen, tok0 + 2 * TOK);  // keys seen by the CTA's last token
  const bool has_b = tok0 + TOK < qlen;  // half B holds a new token (else it is skipped by every role)
  const int nt = (kv_len + 127) / 128;
  const int npages = (kv_len + 15) / 16;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int st = 0; st < kKStages; ++st) {
      mbar_init(bar(kBarKFull + st), 1);
      mbar_init(bar(kBarKFree + st), 1);
    }
    for (int st = 0; st < kVStages; ++st) {
      mbar_init(bar(kBarVFull + st), 1);
      mbar_init(bar(kBarVFree + st), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(kBarSFull + x), 1);
      mbar_init(bar(kBarPFull + x), 128);
      mbar_init(bar(kBarODone + x), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(bar(kBarTmemSlot), kPfTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kSmBar + 8 * kBarTmemSlot);

  if (warp == 0 || warp == 2) {
    // ---------------- TMA producers: warp 0 streams Q and K, warp 2 streams V ----------------
    const bool is_k = warp == 0;
    const int nst = is_k ? kKStages : kVStages;
    const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
    const uint32_t ring = base + (is_k ? kSmK : kSmV);
    const int full0 = is_k ? kBarKFull : kBarVFull, free0 = is_k ? kBarKFree : kBarVFree;
    const int32_t* bt = a.bt + int64_t(seq) * a.bt_stride;
    if (lane == 0) {
      tc::tma_prefetch_desc(tm);
      if (is_k) {
        tc::tma_prefetch_desc(&tm_q);
        mbar_arrive_expect_tx(bar(kBarQ), 2 * kPfTile);
        for (int x = 0; x < 2; ++x) {
          const uint32_t d = base + kSmQ + uint32_t(x) * kPfTile;
          tc::tma_load_3d(d, &tm_q, 0, kvh * G, q0 + tok0 + x * TOK, bar(kBarQ));
          tc::tma_load_3d(d + kPfHalf, &tm_q, 64, kvh * G, q0 + tok0 + x * TOK, bar(kBarQ));
        }
      }
    }
    int issued = 0;  // tiles whose loads were issued
    for (int j = 0; j < nt; ++j) {
      const int st = j % nst, use = j / nst;
      if (j >= nst && !warp_wait(bar(free0 + st), (use - 1) & 1, a.timeout_ns)) break;
      const int p0 = j * 8;
      const int np = min(8, npages - p0);
      int blk = 0;
      if (lane < np) {
        blk = bt[p0 + lane];
        if (blk < 0 || blk >= a.num_blocks) {
          flag(PA_DEV_BAD_BLOCK);
          blk = 0;
        }
      }
      if (lane == 0) mbar_arrive_expect_tx(bar(full0 + st), uint32_t(np) * 4096u);
      for (int p = 0; p < np; ++p) {
        const int b = __shfl_sync(0xffffffffu, blk, p);
        if (lane == 0) {
          const uint32_t d = ring + uint32_t(st) * kPfTile + uint32_t(p) * 2048u;
          tc::tma_load_4d(d, tm, 0, 0, kvh, b, bar(full0 + st));
          tc::tma_load_4d(d + kPfHalf, tm, 64, 0, kvh, b, bar(full0 + st));
        }
      }
      issued = j + 1;
    }
    // Before the CTA may exit, every copy it started must have landed.
    if (is_k) mbar_wait_bounded(bar(kBarQ), 0, a.timeout_ns);
    for (int j = max(0, issued - nst); j < issued; ++j)
      mbar_wait_bounded(bar(full0 + j % nst), (j / nst) & 1, a.timeout_ns);
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t kIdQK = tc::idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t kIdPV = tc::idesc_bf16_f32(128, 128, false, true);
    auto qk = [&](int j, int x) {  // S_x = Q_x K_j^T (lane 0)
      const uint32_t kb = base + kSmK + uint32_t(j % kKStages) * kPfTile;
      const uint32_t qb = base + kSmQ + uint32_t(x) * kPfTile;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = uint32_t(kk >> 2) * kPfHalf + uint32_t(kk & 3) * 32u;
        tc::mma_bf16_ss(tmem + uint32_t(x) * 128u, tc::desc_kmajor(qb + off), tc::desc_kmajor(kb + off), kIdQK,
                        kk > 0);
      }
      tc::commit(bar(kBarSFull + x));
    };
    auto pv = [&](int j, int x) {  // O_x += P_x V_j (lane 0); P_x = first 64 columns of S_x
      const uint32_t vb = base + kSmV + uint32_t(j % kVStages) * kPfTile;
      const uint32_t pt = tmem + uint32_t(x) * 128u;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc::mma_bf16_ts(tmem + kTmO + uint32_t(x) * 128u, pt + uint32_t(kk) * 8u,
                        tc::desc_mnmajor(vb + uint32_t(kk) * 2048u, kPfHalf), kIdPV, j > 0 || kk > 0);
      tc::commit(bar(kBarODone + x));
    };
    bool ok = warp_wait(bar(kBarQ), 0, a.timeout_ns) && warp_wait(bar(kBarKFull), 0, a.timeout_ns);
    if (ok) {
      tc::fence_after_sync();
      if (lane == 0) {
        qk(0, 0);
        if (has_b) qk(0, 1);
        tc::commit(bar(kBarKFree));
      }
      __syncwarp();
    }
    for (int j = 0; ok && j < nt; ++j) {
      const int sv = j % kVStages;
      const bool more = j + 1 < nt;
      if (!(ok = warp_wait(bar(kBarVFull + sv), (j / kVStages) & 1, a.timeout_ns))) break;
      const int valid = kv_len - j * 128;
      if (valid < 128) {
        // Rows past the last key hold stale or never-written values (NaN
        // would survive a zero probability): clear them before P V.
        uint8_t* vs = gbase + kSmV + uint32_t(sv) * kPfTile;
        const int rows = 128 - valid;
        for (int e = lane; e < rows * 16; e += 32) {
          const int r = valid + (e >> 4), c = e & 15;
          *reinterpret_cast<uint4*>(vs + uint32_t(c >> 3) * kPfHalf + uint32_t(r) * 128u + uint32_t(c & 7) * 16u) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
      }
      // half A: P V of this tile, then Q K^T of the next (S_A is free once P_A is consumed, in MMA order)
      if (!(ok = warp_wait(bar(kBarPFull + 0), j & 1, a.timeout_ns))) break;
      tc::fence_after_sync();
      if (lane == 0) pv(j, 0);
      __syncwarp();
      if (more) {
        if (!(ok = warp_wait(bar(kBarKFull + (j + 1) % kKStages), ((j + 1) / kKStages) & 1, a.timeout_ns))) break;
        tc::fence_after_sync();
        if (lane == 0) {
          qk(j + 1, 0);
          if (!has_b) tc::commit(bar(kBarKFree + (j + 1) % kKStages));
        }
        __syncwarp();
      }
      if (!has_b) {
        if (lane == 0) tc::commit(bar(kBarVFree + sv));
        __syncwarp();
        continue;
      }
      // half B, then release the K and V stages
      if (!(ok = warp_wait(bar(kBarPFull + 1), j & 1, a.timeout_ns))) break;
      tc::fence_after_sync();
      if (lane == 0) {
        pv(j, 1);
        tc::commit(bar(kBarVFree + sv));
        if (more) {
          qk(j + 1, 1);
          tc::commit(bar(kBarKFree + (j + 1) % kKStages));
        }
      }
      __syncwarp();
    }
    // No MMA may still run when TMEM is released.
    if (lane == 0) tc::commit(bar(kBarDrain));
    __syncwarp();
    mbar_wait_bounded(bar(kBarDrain), 0, a.timeout_ns);
  } else if (warp >= 4) {
    // ---------------- softmax + epilogue: one query row per thread ----------------
    const int x = (warp - 4) >> 2;  // half
    const bool active = x == 0 || has_b;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // row within the half = TMEM lane
    const int tok = r / G, g = r - (r / G) * G;
    const int qi = tok0 + x * TOK + tok;
    const bool row_valid = qi < qlen;
    const int kmax = row_valid ? c0 + qi + 1 : 0;  // keys [0, kmax) are visible
    const uint32_t tl = tmem + (uint32_t(quad * 32) << 16);
    const uint32_t tS = tl + uint32_t(x) * 128u, tO = tl + kTmO + uint32_t(x) * 128u;
    const float cl = a.scale_log2;
    // Lazy rescaling: the exponent offset m_used (raw logit units) moves only
    // when a row's max exceeds it by more than kRescaleLog2 / cl, so
    // probabilities stay below 2^kRescaleLog2 and O is rarely rescaled; the
    // final division by l uses the same offset, so the result is unchanged.
    constexpr float kRescaleLog2 = 8.f;
    const float thr = kRescaleLog2 / cl;
    float m_used = -INFINITY, l = 0.f;
    bool ok = active;
    for (int j = 0; ok && j < nt; ++j) {
      if (!(ok = warp_wait(bar(kBarSFull + x), j & 1, a.timeout_ns))) break;
      tc::fence_after_sync();
      float s[128];
      __syncwarp();  // tcgen05.ld is warp-collective
      tc::tmem_ld128(tS, s);
      const int lim = kmax - j * 128;  // columns [0, lim) are visible
      if (lim < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = c < lim ? s[c] : -INFINITY;
      }
      float m8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = s[k];
#pragma unroll
      for (int c = 8; c < 128; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
      const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const bool moved = __any_sync(0xffffffffu, mt > m_used + thr);
      float alpha = 1.f;
      if (moved) {
        const float m_new = fmaxf(m_used, mt);
        alpha = m_new == -INFINITY ? 1.f : ex2((m_used - m_new) * cl);  // 0 on a row's first visible tile
        m_used = m_new;
      }
      const float mu = m_used == -INFINITY ? 0.f : m_used * cl;
      float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      // P over the first 64 columns of S, 32 keys (16 columns) at a time:
      // S has been read, and P V of the previous tile, which read the old P,
      // ran before the MMA that produced this S.
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pw[16];
#pragma unroll
        for (int c = ch * 32; c < ch * 32 + 32; c += 2) {
          float e0 = -mu, e1 = -mu;
          ffma2(e0, e1, s[c], s[c + 1], cl, cl);  // s * cl - mu
          if (((c >> 3) & 3) == 3) {              // a quarter of the exponentials on the FMA pipe
            ex2_poly2(e0, e1);
          } else {
            e0 = ex2(e0);
            e1 = ex2(e1);
          }
          pw[(c - ch * 32) >> 1] = pack_bf16x2(e0, e1);
          fadd2(rs[c & 7], rs[(c & 7) + 1], rs[c & 7], rs[(c & 7) + 1], e0, e1);
        }
        tc::tmem_st16(tS + uint32_t(ch) * 16u, pw);
      }
      // O may be rescaled only after P V of the previous tile has completed.
      if (j > 0) {
        if (!(ok = warp_wait(bar(kBarODone + x), (j - 1) & 1, a.timeout_ns))) break;
        tc::fence_after_sync();
        if (moved) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tc::tmem_ld32(tO + uint32_t(c) * 32u, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::tmem_st32(tO + uint32_t(c) * 32u, o);
          }
        }
      }
      tc::tmem_wait_st();
      l = l * alpha + (((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
      tc::fence_before_sync();
      mbar_arrive(bar(kBarPFull + x));
    }
    if (ok) ok = warp_wait(bar(kBarODone + x), (nt - 1) & 1, a.timeout_ns);
    if (ok) {
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* dst = a.out + int64_t(q0 + qi) * a.o_st + int64_t(kvh * G + g) * a.o_sh;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        __syncwarp();
        tc::tmem_ld32(tO + uint32_t(c) * 32u, o);
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(o[8 * v + 0] * inv, o[8 * v + 1] * inv);
            w.y = pack_bf16x2(o[8 * v + 2] * inv, o[8 * v + 3] * inv);
            w.z = pack_bf16x2(o[8 * v + 4] * inv, o[8 * v + 5] * inv);
            w.w = pack_bf16x2(o[8 * v + 6] * inv, o[8 * v + 7] * inv);
            *reinterpret_cast<uint4*>(dst + c * 32 + v * 8) = w;
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kPfTmemCols);
  }
}

}  // namespace pa
