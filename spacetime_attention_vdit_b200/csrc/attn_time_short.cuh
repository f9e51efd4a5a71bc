// attn_time_short.cuh - the time pass of divided attention for short clips.
//
// Divided attention ("Video and 3D Generation" cheatsheet, "Tiny video DiT" and
// "Divided attention"; "Video as a 3D signal", "Patches and attention") first
// runs attention over the T tokens at each spatial site: for every (batch b,
// site s, head h) the tokens {t*HW + s : t < T}.  With T = 21 latent frames each
// such problem is tiny (21 x 21 scores) and there are B*HW*heads of them, so
// the pass moves Q, K, V and O once through HBM at an arithmetic intensity of
// about 10 flop/byte: it is bandwidth-bound, and is built to keep HBM busy.
//
// Design: a producer warp streams problems into a ring of shared-memory stages
// with TMA - one 5-D box per D-block per tensor: {D-block, 1 head, 1 site, TB
// frames, 1 batch} over the view {D, heads, sites, frames, batch}, so the box
// gathers the site's T rows (HW*heads*D elements apart) in one copy and rows
// T .. TB-1 arrive as zeros.  TB is T rounded up to 8 rows, so that as many
// problems as possible fit in shared memory at once (at T = 21, 24-row stages
// hold 10 problems where 32-row ones held 8).  Each consumer group (two warps
// when T > 16, one per 16-row m-tile; one warp otherwise) owns two stages and
// alternates between them, so its next problem is in flight while it computes
// the current one.  A consumer warp computes S = Q K^T and O = P V with
// warp-level bf16 tensor-core MMAs (m16n8k16, fp32 accumulation) on rows padded
// to TP (TB rounded up to 16; the rows TB .. TP-1 that a fragment load reaches
// read rows TB-8 .. TP-9 again: their scores are masked, their probabilities
// are exactly zero and their query rows are never stored), keeps the softmax in
// registers, stages O over the stage's Q rows and writes it with 16-byte
// stores, then releases the stage to the producer.
#pragma once

#include "ptx.cuh"

namespace vdit {

template <int D, int TB>
struct TimeCfg {
  static constexpr int TP = (TB + 15) & ~15;                  // rows and keys padded to 16-row m-tiles
  static constexpr int ROWB = (D * 2 >= 128) ? 128 : D * 2;   // bytes per row of one D-block
  static constexpr int DBLK = ROWB / 2;                       // elements per D-block
  static constexpr int NDB = D / DBLK;                        // D-blocks
  static constexpr int CPB = ROWB / 16;                       // 16-byte chunks per D-block row
  static constexpr int REGION = TB * ROWB;                    // one D-block of one tensor
  static constexpr int TENSOR_BYTES = NDB * REGION;           // = TB * D * 2
  static constexpr int STAGE_BYTES = 3 * TENSOR_BYTES;        // Q, K, V
  static constexpr int WPU = TP >= 32 ? 2 : 1;                // warps per problem (split by 16-row m-tiles)
  // stages: as many as fit in the 227 KB a CTA may use, at most 16, and at most
  // 10 consumer warps at D = 128 so that the registers of the fullest SM
  // sub-partition (three warps of eleven) stay within its 16,384
  static constexpr int MAXW = D >= 128 ? 10 : 16;
  static constexpr int FIT = (231424 / (STAGE_BYTES + 16)) & ~1;
  static constexpr int NSTAGE = FIT < 16 ? (FIT < 2 * (MAXW / WPU) ? FIT : 2 * (MAXW / WPU))
                                         : (16 < 2 * (MAXW / WPU) ? 16 : 2 * (MAXW / WPU));
  static constexpr int NP = NSTAGE / 2;                       // consumer groups, two stages each
  static constexpr int NC = NP * WPU;                         // consumer warps
  static constexpr int THREADS = 32 * (1 + NC);
  // register budget as if the warps filled every sub-partition evenly
  static constexpr int LB_THREADS = 128 * ((1 + NC + 3) / 4);
  static constexpr int SMEM_BYTES = 1024 + NSTAGE * STAGE_BYTES + 2 * NSTAGE * 8;
  static_assert(D % 16 == 0 && D >= 32 && D <= 128, "head_dim");
  static_assert(TB % 8 == 0 && TB >= 8 && TB <= 64, "box rows");
  static_assert(NSTAGE >= 2, "stages");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Byte offset of 16-byte chunk c (0 .. D/8-1) of row r inside one tensor of a
// stage, as the TMA box lays it out: D-block c / CPB, rows of ROWB bytes, the
// chunk index XOR-swizzled with the row (128-byte or 64-byte swizzle).  Rows
// TB .. TP-1 (only when TB is not a multiple of 16) fold back by 8 onto rows
// that the stage holds.
template <int D, int TB>
__device__ __forceinline__ uint32_t time_off(int r, int c) {
  using C = TimeCfg<D, TB>;
  if (TB != C::TP && r >= TB) r -= 8;
  const int key = C::ROWB == 128 ? (r & 7) : ((r >> 1) & 3);
  return (uint32_t)((c / C::CPB) * C::REGION + r * C::ROWB + (((c % C::CPB) ^ key) << 4));
}

// Not volatile: it reads and writes registers only, and the compiler must be
// free to interleave independent accumulation chains with the (volatile)
// shared-memory fragment loads.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct TimeParams {
  __nv_bfloat16* o;
  float* lse;           // may be null; [B, heads, T*HW]
  int B, T, HW, heads;
  float scale_log2;
};

template <int D, int TB>
__global__ void __launch_bounds__(TimeCfg<D, TB>::LB_THREADS, 1)
    attn_time_short_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const TimeParams p) {
  using C = TimeCfg<D, TB>;
  constexpr int TP = C::TP;
  unsigned char* stages = smem_base_1024();
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + C::NSTAGE * C::STAGE_BYTES);
  uint64_t* empty = full + C::NSTAGE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const long long n_units = (long long)p.B * p.HW * p.heads;
  // this CTA's contiguous run of problems
  const long long u_begin = n_units * blockIdx.x / gridDim.x;
  const long long u_end = n_units * (blockIdx.x + 1) / gridDim.x;
  const int n_local = (int)(u_end - u_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::WPU);       // every warp of the consumer group releases the stage
    }
    fence_mbar_init();
  }
  __syncthreads();

  // problem k of this CTA -> stage (k % NP) * 2 + (k / NP) % 2, consumer group k % NP
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;
      // (head, site, batch) of problem u = ((b * HW + s) * heads + h): divided
      // out once, then stepped, so the issue loop carries no division
      int h = (int)(u_begin % p.heads), s, b;
      {
        const long long bs = u_begin / p.heads;
        s = (int)(bs % p.HW);
        b = (int)(bs / p.HW);
      }
      for (int k = 0; k < n_local; ++k) {
        const int st = (k % C::NP) * 2 + ((k / C::NP) & 1);
        const int use = k / (2 * C::NP);                    // earlier fills of this stage
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, 20)) break;
        unsigned char* sb = stages + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
#pragma unroll
        for (int db = 0; db < C::NDB; ++db) {
          tma_load_5d(sb + 0 * C::TENSOR_BYTES + db * C::REGION, &tmQ, &full[st], db * C::DBLK, h, s, 0, b);
          tma_load_5d(sb + 1 * C::TENSOR_BYTES + db * C::REGION, &tmK, &full[st], db * C::DBLK, h, s, 0, b);
          tma_load_5d(sb + 2 * C::TENSOR_BYTES + db * C::REGION, &tmV, &full[st], db * C::DBLK, h, s, 0, b);
        }
        issued = k + 1;
        if (++h == p.heads) {
          h = 0;
          if (++s == p.HW) { s = 0; ++b; }
        }
      }
      // drain: the last fill of every stage has landed before the CTA exits
      for (int k = issued - 2 * C::NP < 0 ? 0 : issued - 2 * C::NP; k < issued; ++k) {
        const int st = (k % C::NP) * 2 + ((k / C::NP) & 1);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[st], (k / (2 * C::NP)) & 1))
          if (globaltimer_ns() - t0 > kWaitLimitNs) { watchdog_trip(21); break; }
      }
    }
    return;
  }

  const int cg = (warp - 1) / C::WPU;       // consumer group
  const int sub = (warp - 1) % C::WPU;      // this warp's m-tiles: sub, sub + WPU, ...
  const int T = p.T;
  const long long row_stride = (long long)p.HW * p.heads * D;    // elements between frames
  const int n_mt = (T + 15) / 16;
  const int g8 = lane >> 2;                  // fragment row within an 8-row group
  const int q2 = (lane & 3) * 2;             // fragment column pair
  int j = 0;                                 // this group's problem count
  // (head, site, batch) of this group's first problem, then stepped by NP
  int h = (int)((u_begin + cg) % p.heads), s, b;
  {
    const long long bs = (u_begin + cg) / p.heads;
    s = (int)(bs % p.HW);
    b = (int)(bs / p.HW);
  }
  for (int k = cg; k < n_local; k += C::NP, ++j) {
    const int st = cg * 2 + (j & 1);
    // every lane of the warp leaves together: the loop body is full of
    // warp-synchronous ldmatrix, mma.sync and shuffles
    if (!warp_wait(&full[st], (j >> 1) & 1, 22)) break;
    unsigned char* sb = stages + st * C::STAGE_BYTES;
    const uint32_t aQ = smem_u32(sb), aK = aQ + C::TENSOR_BYTES, aV = aQ + 2 * C::TENSOR_BYTES;

    for (int mt = sub; mt < n_mt; mt += C::WPU) {
      // ---- S = Q K^T for rows mt*16 .. mt*16+15, all TP key columns
      float sacc[TP / 8][4];
#pragma unroll
      for (int n = 0; n < TP / 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(aQ + time_off<D, TB>(mt * 16 + (lane & 15), kk * 2 + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < TP / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(aK + time_off<D, TB>(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)),
                  b0, b1, b2, b3);
          mma_bf16_16816(sacc[2 * np], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(sacc[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      // ---- softmax over the T valid keys of rows g8 and g8 + 8
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < TP / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool valid = n * 8 + q2 + e < T;
          if (!valid) { sacc[n][e] = -INFINITY; sacc[n][2 + e] = -INFINITY; }
          mx0 = fmaxf(mx0, sacc[n][e]);
          mx1 = fmaxf(mx1, sacc[n][2 + e]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float m0 = mx0 * p.scale_log2, m1 = mx1 * p.scale_log2;
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int n = 0; n < TP / 8; ++n) {
        sacc[n][0] = ex2_approx(fmaf(sacc[n][0], p.scale_log2, -m0));
        sacc[n][1] = ex2_approx(fmaf(sacc[n][1], p.scale_log2, -m0));
        sacc[n][2] = ex2_approx(fmaf(sacc[n][2], p.scale_log2, -m1));
        sacc[n][3] = ex2_approx(fmaf(sacc[n][3], p.scale_log2, -m1));
        l0 += sacc[n][0] + sacc[n][1];
        l1 += sacc[n][2] + sacc[n][3];
      }
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

      // ---- O = P V (P straight from the S accumulators, rounded to bf16)
      float oacc[D / 8][4];
#pragma unroll
      for (int n = 0; n < D / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
#pragma unroll
      for (int k2 = 0; k2 < TP / 16; ++k2) {
        const uint32_t a0 = pack_bf16x2(sacc[2 * k2][0], sacc[2 * k2][1]);
        const uint32_t a1 = pack_bf16x2(sacc[2 * k2][2], sacc[2 * k2][3]);
        const uint32_t a2 = pack_bf16x2(sacc[2 * k2 + 1][0], sacc[2 * k2 + 1][1]);
        const uint32_t a3 = pack_bf16x2(sacc[2 * k2 + 1][2], sacc[2 * k2 + 1][3]);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(aV + time_off<D, TB>(k2 * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), dp * 2 + (lane >> 4)),
                    b0, b1, b2, b3);
          mma_bf16_16816(oacc[2 * dp], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(oacc[2 * dp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      // ---- normalise; stage rows < T of this m-tile over their (consumed) Q rows
      __syncwarp();
      const float inv0 = 1.f / l0, inv1 = 1.f / l1;
      const int r0 = mt * 16 + g8, r1 = r0 + 8;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {       // 8 columns = one 16-byte chunk
        if (r0 < T)
          *reinterpret_cast<uint32_t*>(sb + time_off<D, TB>(r0, n) + q2 * 2) =
              pack_bf16x2(oacc[n][0] * inv0, oacc[n][1] * inv0);
        if (r1 < T)
          *reinterpret_cast<uint32_t*>(sb + time_off<D, TB>(r1, n) + q2 * 2) =
              pack_bf16x2(oacc[n][2] * inv1, oacc[n][3] * inv1);
      }
      if (p.lse != nullptr && (lane & 3) == 0) {
        const long long lbase = ((long long)b * p.heads + h) * ((long long)T * p.HW) + s;
        if (r0 < T) p.lse[lbase + (long long)r0 * p.HW] = (m0 + __log2f(l0)) * 0.69314718055994531f;
        if (r1 < T) p.lse[lbase + (long long)r1 * p.HW] = (m1 + __log2f(l1)) * 0.69314718055994531f;
      }
      __syncwarp();
    }

    // ---- write this warp's O rows back to their tokens, then hand the stage back
    const long long first = (((long long)b * T * p.HW + s) * p.heads + h) * D;   // element of t = 0
    for (int mt = sub; mt < n_mt; mt += C::WPU) {
      const int rows = min(16, T - mt * 16);
      for (int i = lane; i < rows * (D / 8); i += 32) {
        const int t = mt * 16 + i / (D / 8), c = i % (D / 8);
        const uint4 val = *reinterpret_cast<const uint4*>(sb + time_off<D, TB>(t, c));
        *reinterpret_cast<uint4*>(p.o + first + t * row_stride + c * 8) = val;
      }
    }
    // the stage's next fill is an async-proxy write over these generic-proxy accesses
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    for (h += C::NP; h >= p.heads;) {
      h -= p.heads;
      if (++s == p.HW) { s = 0; ++b; }
    }
  }
}

}  // namespace vdit
