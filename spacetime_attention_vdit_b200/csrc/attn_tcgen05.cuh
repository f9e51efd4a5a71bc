// attn_tcgen05.cuh - fused flash-style attention forward on the 5th-generation
// tensor cores (tcgen05 + TMEM), TMA-staged Q/K/V tiles.
//
// Computes O = softmax(scale * Q K^T) V per (sequence, head), non-causal: the
// full 3D self-attention of "How AI Generates Video: Inside Sora and Wan2.1 on
// a Real GPU" (section 5: every token attends to every token; section 7: logits
// scaled by 1/sqrt(head_dim)), tiled so that the L x L scores never leave the
// SM ("Video Diffusion Models, in depth", Step 3).  The same kernel runs the
// space pass of divided attention (each frame is a contiguous sequence) and,
// through a strided tensor map, a time pass with long sequences.
//
// One CTA computes one 128-row query tile of one (sequence, head):
//   warp 0      TMA producer: Q once, then K_j and V_j into an NSTAGE ring;
//   warp 1      allocates TMEM and issues the UMMAs (one thread):
//                 S_j = Q K_j^T into one of two TMEM score buffers,
//                 O  += P_j V_j into the TMEM accumulator;
//   warps 2..5  softmax, one query row per thread (TMEM lane = row): read S_j,
//               running max (kept unless it grows by more than 2^8, an exact
//               rescaling rule), P_j = 2^(s*scale*log2e - m) rounded to bf16
//               into shared memory, O rescaled in TMEM when the max moved,
//               and finally O / l to global memory with the row's log-sum-exp.
// S_{j+1} is computed on the tensor cores while the softmax works on S_j.
#pragma once

#include <math.h>

#include "ptx.cuh"

namespace vdit {

template <int D>
struct AttnCfg {
  static constexpr int BM = 128;                               // query rows per tile
  static constexpr int BN = 128;                               // keys per KV tile
  static constexpr int ROWB = (D * 2 >= 128) ? 128 : D * 2;    // bytes per staged row of one D-block
  static constexpr int DBLK = ROWB / 2;                        // elements per D-block
  static constexpr int NDB = D / DBLK;                         // D-blocks per tile
  static constexpr uint32_t SWZ = ROWB == 128 ? kSwizzle128 : (ROWB == 64 ? kSwizzle64 : kSwizzle32);
  static constexpr int DB_BYTES = BM * ROWB;                   // one D-block of a 128-row tile
  static constexpr int TILE_BYTES = BM * D * 2;
  static constexpr int NSTAGE = D >= 128 ? 2 : (D >= 64 ? 3 : 4);
  static constexpr int P_BYTES = BM * BN * 2;
  static constexpr int NBARS = 1 + 3 * NSTAGE + 2 + 2 + 1 + 1 + 1;
  static constexpr int SMEM_BYTES = 1024 + TILE_BYTES + 2 * NSTAGE * TILE_BYTES + P_BYTES + NBARS * 8 + 16;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;                         // S buffers at columns 0 and 128
  static constexpr uint32_t O_COL = 256;                       // O accumulator, D columns
  static constexpr uint32_t IDESC_QK = umma_idesc_bf16(BM, BN, 0, 0);  // Q, K both K-major
  static constexpr uint32_t IDESC_PV = umma_idesc_bf16(BM, D, 0, 1);   // P K-major, V MN-major
  static_assert(D % 16 == 0 && D >= 32 && D <= 128, "head_dim");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Where a (sequence bb, position i) lives among the caller's tokens.
//   kSeq : sequence bb = b*grp + t holds the contiguous tokens [bb*L, bb*L + L)
//          (full attention: grp = 1; space pass: grp = frames per clip).
//   kTime: sequence bb = b*grp + s holds tokens {b*L*grp + i*grp + s} (time pass:
//          grp = sites per frame, L = frames).
enum AttnMode : int { kSeq = 0, kTime = 1 };

struct AttnParams {
  __nv_bfloat16* o;
  float* lse;          // may be null
  int n_seq;           // sequences
  int L;               // tokens per sequence
  int heads;
  int grp;             // see AttnMode
  int mode;
  int n_qtiles;        // ceil(L / 128)
  int n_kv;            // ceil(L / 128)
  float scale_log2;    // scale * log2(e)
};

// Wait sites recorded by the watchdog.
enum : int {
  kSiteQFull = 1, kSiteKFull, kSiteVFull, kSiteKvEmpty, kSiteSFull, kSiteSFree, kSitePFull, kSiteODone,
  kSiteDrain
};

// A wait bounded by time only (used to drain copies and MMAs before exit).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) { watchdog_trip(kSiteDrain); return; }
  }
}

// All 32 lanes wait; the result is made warp-uniform, so that a lane whose
// wait ran out never leaves its warp-mates inside a .sync.aligned instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int site) {
  const bool ok = mbar_wait(bar, parity, site);
  return __all_sync(0xffffffffu, ok) != 0;
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_tcgen05_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<D>;
  unsigned char* smem_raw = dyn_smem;
  const uintptr_t base = (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023);
  unsigned char* sQ = reinterpret_cast<unsigned char*>(base);
  unsigned char* sK = sQ + C::TILE_BYTES;
  unsigned char* sV = sK + C::NSTAGE * C::TILE_BYTES;
  unsigned char* sP = sV + C::NSTAGE * C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + C::P_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* v_full = k_full + C::NSTAGE;
  uint64_t* kv_empty = v_full + C::NSTAGE;
  uint64_t* s_full = kv_empty + C::NSTAGE;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int tile = blockIdx.x;
  const int qt = tile % p.n_qtiles;
  const int bh = tile / p.n_qtiles;
  const int h = bh % p.heads;
  const int bb = bh / p.heads;
  const int q0 = qt * C::BM;
  // tensor-map coordinates of this sequence: (d, head, site, position, batch)
  const int c_site = p.mode == kTime ? bb % p.grp : 0;
  const int c_batch = p.mode == kTime ? bb / p.grp : bb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
#pragma unroll
      for (int db = 0; db < C::NDB; ++db)
        tma_load_5d(sQ + db * C::DB_BYTES, &tmQ, q_full, db * C::DBLK, h, c_site, q0, c_batch);
      int issued = 0;
      for (int j = 0; j < p.n_kv; ++j) {
        const int st = j % C::NSTAGE;
        if (j >= C::NSTAGE && !mbar_wait(&kv_empty[st], ((j / C::NSTAGE) - 1) & 1, kSiteKvEmpty)) break;
        mbar_arrive_expect_tx(&k_full[st], C::TILE_BYTES);
#pragma unroll
        for (int db = 0; db < C::NDB; ++db)
          tma_load_5d(sK + st * C::TILE_BYTES + db * C::DB_BYTES, &tmK, &k_full[st], db * C::DBLK, h, c_site,
                      j * C::BN, c_batch);
        mbar_arrive_expect_tx(&v_full[st], C::TILE_BYTES);
#pragma unroll
        for (int db = 0; db < C::NDB; ++db)
          tma_load_5d(sV + st * C::TILE_BYTES + db * C::DB_BYTES, &tmV, &v_full[st], db * C::DBLK, h, c_site,
                      j * C::BN, c_batch);
        issued = j + 1;
      }
      // No copy may still be landing in shared memory when the CTA exits.
      mbar_drain(q_full, 0);
      for (int j = issued - C::NSTAGE < 0 ? 0 : issued - C::NSTAGE; j < issued; ++j) {
        const int st = j % C::NSTAGE;
        mbar_drain(&k_full[st], (j / C::NSTAGE) & 1);
        mbar_drain(&v_full[st], (j / C::NSTAGE) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sPa = smem_u32(sP);
      constexpr uint32_t SBO = 8 * C::ROWB;       // 8-row core-matrix group stride
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj % C::NSTAGE;
        if (!mbar_wait(&v_full[st], (jj / C::NSTAGE) & 1, kSiteVFull)) return false;
        if (!mbar_wait(p_full, jj & 1, kSitePFull)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          // A = P (128 x 16 keys), K-major, 128-byte swizzle, 64 keys per 16 KB block
          const uint64_t a = umma_sdesc(sPa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSwizzle128);
          // B = V (16 keys x D), MN-major: D-blocks DB_BYTES apart, 8-key groups SBO apart
          const uint64_t b = umma_sdesc(sVa + st * C::TILE_BYTES + kk * 16 * C::ROWB, C::DB_BYTES, SBO, C::SWZ);
          umma_ss(tmem + C::O_COL, a, b, C::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[st]);
        umma_commit(o_done);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, kSiteQFull);
      for (int j = 0; j < p.n_kv && ok; ++j) {
        const int st = j % C::NSTAGE;
        const int sb = j & 1;
        if (!mbar_wait(&k_full[st], (j / C::NSTAGE) & 1, kSiteKFull)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1, kSiteSFree)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / (C::DBLK / 16)) * C::DB_BYTES + (kk % (C::DBLK / 16)) * 32;
          const uint64_t a = umma_sdesc(sQa + off, 16, SBO, C::SWZ);
          const uint64_t b = umma_sdesc(sKa + st * C::TILE_BYTES + off, 16, SBO, C::SWZ);
          umma_ss(tmem + C::S_COL + sb * C::BN, a, b, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[sb]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(p.n_kv - 1);
      // every UMMA issued above has finished before TMEM is released
      umma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- softmax
    const int quad = warp & 3;                    // TMEM lanes this warp may touch
    const int row = quad * 32 + lane;             // query row within the tile
    const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
    float m_use = -INFINITY;                      // max used for the exponentials (log2 units)
    float l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < p.n_kv; ++j) {
      const int sb = j & 1;
      if (!warp_wait(&s_full[sb], (j >> 1) & 1, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tlane + C::S_COL + sb * C::BN + c * 32, s[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&s_free[sb]);

      const int valid = p.L - j * C::BN;          // keys of this tile inside the sequence
      if (valid < C::BN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e >= valid) s[c][e] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(s[c][e]));
      const float m_new = mx * p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_use = m_new;
      } else if (m_new > m_use + 8.f) {
        alpha = ex2_approx(m_use - m_new);
        m_use = m_new;
        rescale = true;
      }
      const float neg_m = -m_use;
      float rsum = 0.f;
      uint32_t pk[64];                            // P row as bf16 pairs
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[c][e]), p.scale_log2, neg_m));
          const float p1 = ex2_approx(fmaf(__uint_as_float(s[c][e + 1]), p.scale_log2, neg_m));
          rsum += p0 + p1;
          pk[(c * 32 + e) >> 1] = pack_bf16x2(p0, p1);
        }

      // P and O may be touched only once the previous P.V product is done.
      if (j >= 1 && !warp_wait(o_done, (j - 1) & 1, kSiteODone)) { ok = false; break; }
      tc_fence_after();
      // P row -> shared memory, K-major, 128-byte swizzle: key block kb (64 keys,
      // 16 KB), 16-byte chunk c of the row stored at chunk c ^ (row % 8).
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int kb = ch >> 3, c = ch & 7;
        uint4* dst = reinterpret_cast<uint4*>(sP + kb * 16384 + row * 128 + ((c ^ (row & 7)) << 4));
        *dst = make_uint4(pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tlane + C::O_COL + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tlane + C::O_COL + c * 32, o);
        }
        tmem_st_wait();
      }
      l_sum = l_sum * alpha + rsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }

    // ------------------------------------------------------------- epilogue
    if (ok && warp_wait(o_done, (p.n_kv - 1) & 1, kSiteODone)) {
      tc_fence_after();
      const int i = q0 + row;                     // position in the sequence
      const float inv_l = 1.f / l_sum;
      long long token;
      if (p.mode == kTime) {
        const int b = bb / p.grp, sidx = bb % p.grp;
        token = (long long)b * p.L * p.grp + (long long)i * p.grp + sidx;
      } else {
        token = (long long)bb * p.L + i;
      }
      __nv_bfloat16* orow = p.o + (token * p.heads + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tlane + C::O_COL + c * 32, o);
        tmem_ld_wait();
        if (i < p.L) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + c * 32 + e) = v;
          }
        }
      }
      if (p.lse != nullptr && i < p.L) {
        const int b = bb / p.grp, g = bb % p.grp;
        const long long pos = p.mode == kTime ? (long long)i * p.grp + g : (long long)g * p.L + i;
        p.lse[((long long)b * p.heads + h) * ((long long)p.L * p.grp) + pos] =
            (m_use + __log2f(l_sum)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace vdit
