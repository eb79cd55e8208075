// Byte-moving kernels of the paged KV cache (sm_100a): the per-token cache
// write by slot (plain, or quantizing into an FP8 cache), the whole-block
// copy of copy-on-write, and the block swap between the device pool and a
// pinned host pool.  The pages fix what these do without naming kernels: a
// new token's K/V lands in the physical block its table names, at its
// offset in that block, and a write into a block that several samples share
// first copies the block (vLLM launch blog, "PagedAttention" section, as
// summarised on the CSDN discovery note, item 2); blocks can be swapped out
// (agientry.com overview, opening section).
//
// Both are pure HBM traffic.  Every (token, kv head) row of K or V is
// head_size * elem bytes (256 B for bf16/128 and fp32/64) and contiguous on
// both sides in the layout [num_blocks, num_kv_heads, 16, head_size], so a
// thread moves one 16-byte vector and 16 consecutive lanes move one row
// with fully coalesced loads and stores.
#pragma once

#include "pa_common.cuh"

namespace pa {

// Cache write: for token t, head h, vector c of the row:
//   k_cache[slot / 16, h, slot % 16, c] = key[t, h, c]   (same for V)
// slot == -1 skips the token; any other slot outside [0, num_slots) sets
// PA_DEV_BAD_SLOT and skips it.  Strides are in 16-byte vectors.
template <int VPR>  // 16-byte vectors per row
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const uint4* __restrict__ key,
                                                                const uint4* __restrict__ value, uint4* kc,
                                                                uint4* vc, const int64_t* __restrict__ slots,
                                                                int64_t T, int Hkv, int64_t k_st, int64_t k_sh,
                                                                int64_t v_st, int64_t v_sh, int64_t num_slots) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t per_tok = int64_t(Hkv) * VPR;
  const int64_t total = T * per_tok;
  const int64_t step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total; idx += step) {
    const int64_t t = idx / per_tok;
    const int r = int(idx - t * per_tok);
    const int h = r / VPR, c = r % VPR;
    const int64_t s = slots[t];
    if (s == -1) continue;
    if (s < -1 || s >= num_slots) {
      if (h == 0 && c == 0) flag(PA_DEV_BAD_SLOT);
      continue;
    }
    const int64_t dst = (((s >> 4) * Hkv + h) * 16 + (s & 15)) * VPR + c;
    const uint4 kv = ld_nc_v4(key + t * k_st + h * k_sh + c);
    const uint4 vv = ld_nc_v4(value + t * v_st + h * v_sh + c);
    kc[dst] = kv;
    vc[dst] = vv;
  }
}

// Cache write into an FP8 (e4m3) cache: the same scatter, but each value is
// stored as the e4m3 code of float(x) / scale[h] (IEEE fp32 division, round
// to nearest even, saturating).  A thread produces one 16-byte vector of 16
// codes from 16 input elements.  Strides are in input elements.
template <typename Tin, int OPR>  // OPR: 16-byte code vectors per row (head_size / 16)
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const Tin* __restrict__ key, const Tin* __restrict__ value, uint4* kc, uint4* vc,
    const int64_t* __restrict__ slots, int64_t T, int Hkv, int64_t k_st, int64_t k_sh, int64_t v_st,
    int64_t v_sh, int64_t num_slots, const float* __restrict__ k_scale, const float* __restrict__ v_scale) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int EPQ = 16 / int(sizeof(Tin));
  const int64_t per_tok = int64_t(Hkv) * OPR;
  const int64_t total = T * per_tok;
  const int64_t step = int64_t(gridDim.x) * blockDim.x;
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total; idx += step) {
    const int64_t t = idx / per_tok;
    const int r = int(idx - t * per_tok);
    const int h = r / OPR, c = r % OPR;
    const int64_t s = slots[t];
    if (s == -1) continue;
    if (s < -1 || s >= num_slots) {
      if (h == 0 && c == 0) flag(PA_DEV_BAD_SLOT);
      continue;
    }
    float kf[16], vf[16];
    const uint4* kp = reinterpret_cast<const uint4*>(key + t * k_st + h * k_sh + c * 16);
    const uint4* vp = reinterpret_cast<const uint4*>(value + t * v_st + h * v_sh + c * 16);
#pragma unroll
    for (int v = 0; v < 16 / EPQ; ++v) {
      Elem<Tin>::unpack(ld_nc_v4(kp + v), kf + v * EPQ);
      Elem<Tin>::unpack(ld_nc_v4(vp + v), vf + v * EPQ);
    }
    const float ks = k_scale[h], vs = v_scale[h];
    uint32_t kw[4], vw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kw[i] = quantize_e4m3x2(__fdiv_rn(kf[4 * i], ks), __fdiv_rn(kf[4 * i + 1], ks)) |
              (quantize_e4m3x2(__fdiv_rn(kf[4 * i + 2], ks), __fdiv_rn(kf[4 * i + 3], ks)) << 16);
      vw[i] = quantize_e4m3x2(__fdiv_rn(vf[4 * i], vs), __fdiv_rn(vf[4 * i + 1], vs)) |
              (quantize_e4m3x2(__fdiv_rn(vf[4 * i + 2], vs), __fdiv_rn(vf[4 * i + 3], vs)) << 16);
    }
    const int64_t dst = (((s >> 4) * Hkv + h) * 16 + (s & 15)) * OPR + c;
    kc[dst] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
    vc[dst] = make_uint4(vw[0], vw[1], vw[2], vw[3]);
  }
}

// Copy-on-write: for each pair (src, dst) copy the whole block, K and V.
// block_vecs = num_kv_heads * 16 * head_size * elem / 16.  grid.y strides
// over pairs, grid.x over the block's vectors.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* kc, uint4* vc, const int64_t* __restrict__ pairs,
                                                          int64_t n, int64_t block_vecs, int64_t num_blocks) {
  pdl_wait();
  pdl_launch_dependents();
  for (int64_t p = blockIdx.y; p < n; p += gridDim.y) {
    const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (blockIdx.x == 0 && threadIdx.x == 0) flag(PA_DEV_BAD_BLOCK);
      continue;
    }
    const uint4* ks = kc + src * block_vecs;
    const uint4* vs = vc + src * block_vecs;
    uint4* kd = kc + dst * block_vecs;
    uint4* vd = vc + dst * block_vecs;
    for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < block_vecs;
         v += int64_t(gridDim.x) * blockDim.x) {
      const uint4 a = ks[v];
      const uint4 b = vs[v];
      kd[v] = a;
      vd[v] = b;
    }
  }
}

// Swap copy: whole blocks from one pool to another (device <-> pinned host,
// reached through unified addressing).  For each pair (src, dst):
// dst_k[dst] = src_k[src], dst_v[dst] = src_v[src]; ids outside their pool
// set PA_DEV_BAD_BLOCK and are skipped.
__global__ void __launch_bounds__(256) swap_blocks_kernel(const uint4* sk, const uint4* sv, uint4* dk, uint4* dv,
                                                          const int64_t* __restrict__ pairs, int64_t n,
                                                          int64_t block_vecs, int64_t n_src, int64_t n_dst) {
  pdl_wait();
  pdl_launch_dependents();
  for (int64_t p = blockIdx.y; p < n; p += gridDim.y) {
    const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= n_src || dst < 0 || dst >= n_dst) {
      if (blockIdx.x == 0 && threadIdx.x == 0) flag(PA_DEV_BAD_BLOCK);
      continue;
    }
    const uint4* ks = sk + src * block_vecs;
    const uint4* vs = sv + src * block_vecs;
    uint4* kd = dk + dst * block_vecs;
    uint4* vd = dv + dst * block_vecs;
    for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < block_vecs;
         v += int64_t(gridDim.x) * blockDim.x) {
      const uint4 a = ks[v];
      const uint4 b = vs[v];
      kd[v] = a;
      vd[v] = b;
    }
  }
}

// One warp waits on a barrier that nothing completes; the bounded wait must
// give up and set PA_DEV_TIMEOUT.  No copy is in flight.
__global__ void wait_selftest_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncwarp();
  mbar_wait_bounded(smem_u32(&bar), 0, timeout_ns);
}

}  // namespace pa
