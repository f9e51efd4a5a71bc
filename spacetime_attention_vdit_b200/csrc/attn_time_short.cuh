// attn_time_short.cuh - the time pass of divided attention for short clips.
//
// Divided attention ("Video and 3D Generation" cheatsheet, "Tiny video DiT" and
// "Divided attention"; "Video as a 3D signal", "Patches and attention") first
// runs attention over the T tokens at each spatial site: for every (batch b,
// site s, head h) the tokens {t*HW + s : t < T}.  With T = 21 latent frames each
// such problem is tiny (21 x 21 scores) and there are B*HW*heads of them, so
// the pass moves Q, K, V and O once through HBM at an arithmetic intensity of
// about 10 flop/byte: it is bandwidth-bound, not tensor-bound.
//
// Design: one warp owns one (b, s, h) problem at a time.  It copies the T rows of
// Q, K and V (each row is one head's 256 contiguous bytes; rows are HW*heads*D
// elements apart) into its own swizzled shared-memory slots with 16-byte
// cp.async, computes S = Q K^T and O = P V with warp-level bf16 tensor-core
// MMAs (m16n8k16, fp32 accumulation) on rows padded to TP, keeps the softmax in
// registers, stages O back through shared memory and writes it with 16-byte
// stores.  Eight warps per CTA (fewer when T > 32) keep the other problems'
// loads in flight while one computes; consecutive warps take consecutive heads of the same site, so a CTA
// streams contiguous runs of each token row.  Pad rows of K and V are zero.
#pragma once

#include "ptx.cuh"

namespace vdit {

template <int D, int TP>
struct TimeCfg {
  static constexpr int CPR = D / 8;                          // 16-byte chunks per row
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int SLOT_BYTES = TP * ROW_BYTES;          // one tensor's rows
  static constexpr int WARP_BYTES = 3 * SLOT_BYTES;          // Q, K, V
  // eight warps when their slots fit in 200 KB, fewer for long padded rows
  static constexpr int WARPS = (200 * 1024) / WARP_BYTES >= 8 ? 8 : (200 * 1024) / WARP_BYTES;
  static constexpr int SMEM_BYTES = WARPS * WARP_BYTES;
  static_assert(D % 16 == 0 && D >= 32 && D <= 128, "head_dim");
  static_assert(TP == 16 || TP == 32 || TP == 64, "padded length");
};

// Physical 16-byte chunk of logical chunk c in row r: XOR-swizzled so that the
// eight rows an ldmatrix reads at one column fall in different banks.
template <int D>
__device__ __forceinline__ int time_swz(int r, int c) {
  if constexpr (D / 8 >= 8) return c ^ (r & 7);
  else return c ^ ((r >> 1) & 3);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct TimeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* o;
  float* lse;           // may be null; [B, heads, T*HW]
  int B, T, HW, heads;
  float scale_log2;
};

template <int D, int TP>
__global__ void __launch_bounds__(256) attn_time_short_kernel(const TimeParams p) {
  using C = TimeCfg<D, TP>;
  unsigned char* smem_raw = dyn_smem;
  if (watchdog_tripped()) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wbase = smem_raw + warp * C::WARP_BYTES;
  unsigned char* sQ = wbase;
  unsigned char* sK = wbase + C::SLOT_BYTES;
  unsigned char* sV = wbase + 2 * C::SLOT_BYTES;
  const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);

  // zero the whole slot once: rows >= T stay zero for every problem
  for (int i = lane; i < C::WARP_BYTES / 16; i += 32)
    reinterpret_cast<uint4*>(wbase)[i] = make_uint4(0, 0, 0, 0);
  __syncwarp();

  const int T = p.T;
  const long long n_units = (long long)p.B * p.HW * p.heads;
  const long long row_stride = (long long)p.HW * p.heads * D;    // elements between frames
  const int n_mt = (T + 15) / 16;

  for (long long u = (long long)blockIdx.x * C::WARPS + warp; u < n_units;
       u += (long long)gridDim.x * C::WARPS) {
    const int h = (int)(u % p.heads);
    const long long bs = u / p.heads;
    const int s = (int)(bs % p.HW);
    const int b = (int)(bs / p.HW);
    const long long first = (((long long)b * T * p.HW + s) * p.heads + h) * D;  // element of (t = 0)

    // ---- load T rows of Q, K, V
    for (int i = lane; i < T * C::CPR; i += 32) {
      const int t = i / C::CPR, c = i - t * C::CPR;
      const long long g = first + t * row_stride + c * 8;
      const uint32_t so = t * C::ROW_BYTES + (time_swz<D>(t, c) << 4);
      cp_async16(aQ + so, p.q + g);
      cp_async16(aK + so, p.k + g);
      cp_async16(aV + so, p.v + g);
    }
    cp_async_wait_all();
    __syncwarp();

    const int g8 = lane >> 2;           // fragment row within an 8-row group
    const int q2 = (lane & 3) * 2;      // fragment column pair
    for (int mt = 0; mt < n_mt; ++mt) {
      // ---- S = Q K^T for rows mt*16 .. mt*16+15, all TP key columns
      float sacc[TP / 8][4];
#pragma unroll
      for (int n = 0; n < TP / 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        {
          const int r = mt * 16 + (lane & 15), c = kk * 2 + (lane >> 4);
          ldsm_x4(aQ + r * C::ROW_BYTES + (time_swz<D>(r, c) << 4), a0, a1, a2, a3);
        }
#pragma unroll
        for (int np = 0; np < TP / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3), c = kk * 2 + ((lane >> 3) & 1);
          ldsm_x4(aK + r * C::ROW_BYTES + (time_swz<D>(r, c) << 4), b0, b1, b2, b3);
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
          const int r = k2 * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), c = dp * 2 + (lane >> 4);
          ldsm_x4_t(aV + r * C::ROW_BYTES + (time_swz<D>(r, c) << 4), b0, b1, b2, b3);
          mma_bf16_16816(oacc[2 * dp], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(oacc[2 * dp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      // ---- normalise, stage rows < T of this m-tile over their (consumed) Q rows
      __syncwarp();
      const float inv0 = 1.f / l0, inv1 = 1.f / l1;
      const int r0 = mt * 16 + g8, r1 = r0 + 8;
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        const int c = n;                        // 8 columns = one 16-byte chunk
        if (r0 < T)
          *reinterpret_cast<uint32_t*>(sQ + r0 * C::ROW_BYTES + (time_swz<D>(r0, c) << 4) + q2 * 2) =
              pack_bf16x2(oacc[n][0] * inv0, oacc[n][1] * inv0);
        if (r1 < T)
          *reinterpret_cast<uint32_t*>(sQ + r1 * C::ROW_BYTES + (time_swz<D>(r1, c) << 4) + q2 * 2) =
              pack_bf16x2(oacc[n][2] * inv1, oacc[n][3] * inv1);
      }
      if (p.lse != nullptr && (lane & 3) == 0) {
        const long long lbase = ((long long)b * p.heads + h) * ((long long)T * p.HW) + s;
        if (r0 < T) p.lse[lbase + (long long)r0 * p.HW] = (m0 + __log2f(l0)) * 0.69314718055994531f;
        if (r1 < T) p.lse[lbase + (long long)r1 * p.HW] = (m1 + __log2f(l1)) * 0.69314718055994531f;
      }
      __syncwarp();
    }

    // ---- write O rows back to their tokens
    for (int i = lane; i < T * C::CPR; i += 32) {
      const int t = i / C::CPR, c = i - t * C::CPR;
      const uint4 val = *reinterpret_cast<const uint4*>(sQ + t * C::ROW_BYTES + (time_swz<D>(t, c) << 4));
      *reinterpret_cast<uint4*>(p.o + first + t * row_stride + c * 8) = val;
    }
    __syncwarp();
  }
}

}  // namespace vdit
