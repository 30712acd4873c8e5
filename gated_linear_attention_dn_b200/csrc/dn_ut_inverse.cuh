// The 64x64 unit-lower-triangular inverse of the UT transform, T = (I + A)^{-1},
// shared by the chunk kernels. fp32 on the CUDA cores with TF32 warp tensor-core
// products for the block merges; it writes T as bf16 operand tiles for tcgen05.
// Callers pass the warp count of the group that runs it and the hardware barrier
// that group synchronises on, so it can run on a whole CTA or on one warp group
// while other warps of the CTA do something else.
#pragma once

#include "dn_tc_ptx.cuh"

namespace dn {
namespace ut {

using tc::canon;
using tc::pack_bf16;

// Index into a 64x64 fp32 array: rows of 64, columns XOR-permuted in groups of 4
// by (row mod 8), so float4 accesses stay aligned and column walks by
// consecutive rows spread over the banks.
__device__ __forceinline__ int xi(int r, int c) { return (r << 6) | (c ^ ((r & 7) << 2)); }

// bar.sync on hardware barrier `id` for `count` threads (a warp-group-local __syncthreads).
__device__ __forceinline__ void group_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier `id` over `count` threads that also returns whether any of them passed pred = true.
__device__ __forceinline__ bool group_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// Warp-level tensor-core product (mma.sync, TF32 inputs, fp32 accumulation), used only for the
// small block products inside the triangular inverse; T is rounded to bf16 afterwards, so TF32
// (10-bit mantissa) operands here add an error well below that rounding. Fragment layouts of
// m16n8k8 row.col (g = lane / 4, t = lane % 4): A 16x8: (g, t) (g+8, t) (g, t+4) (g+8, t+4);
// B 8x8: (t, g) (t+4, g); C 16x8: (g, 2t) (g, 2t+1) (g+8, 2t) (g+8, 2t+1).
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void mma_tf32(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// d[16x8] += X[16 x K] * Y[K x 8] for one warp; X(i, k), Y(k, n) fetch elements.
template <int K, class FX, class FY>
__device__ __forceinline__ void warp_mm(float* d, FX X, FY Y, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int k = 0; k < K; k += 8) {
    const uint32_t av[4] = {to_tf32(X(g, k + t)), to_tf32(X(g + 8, k + t)), to_tf32(X(g, k + t + 4)),
                            to_tf32(X(g + 8, k + t + 4))};
    const uint32_t bv[2] = {to_tf32(Y(k + t, g)), to_tf32(Y(k + t + 4, g))};
    mma_tf32(d, av, bv);
  }
}

// writes the 16x8 accumulator fragment as column pairs through W(i, n, v_n, v_n+1)
template <class FW>
__device__ __forceinline__ void warp_store2(const float* d, FW W, int lane) {
  const int g = lane >> 2, t = lane & 3;
  W(g, 2 * t, d[0], d[1]);
  W(g + 8, 2 * t, d[2], d[3]);
}

// writes the 16x8 accumulator fragment through W(i, n, value)
template <class FW>
__device__ __forceinline__ void warp_store(const float* d, FW W, int lane) {
  const int g = lane >> 2, t = lane & 3;
  W(g, 2 * t, d[0]);
  W(g, 2 * t + 1, d[1]);
  W(g + 8, 2 * t, d[2]);
  W(g + 8, 2 * t + 1, d[3]);
}

// T = (I + L)^{-1} for the 64x64 strictly lower L in sL (zeros on and above the diagonal), run
// by NW >= 4 warps (threads tid = 0 .. 32 NW - 1 of the calling group, which synchronises on
// hardware barrier `bar_id`; all of them call it).
// Blocking by doubling: the eight 8x8 diagonal blocks by forward substitution (one column per
// thread, chains of at most seven steps); then three merge levels with warp mma.sync, each using
// [[A, 0], [C, B]]^{-1} = [[A^-1, 0], [-B^-1 C A^-1, B^-1]]:
//   8 -> 16 (warps 0..3), 16 -> 32 (warps 0..3), 32 -> 64 (eight 16x8 tiles over the NW warps).
// fp32 blocks that later levels read are kept in sT; every element of the lower triangle is also
// written as bf16 straight into rows 0..63 of the K-major tile tp (scaled by column factor
// cs_c[i] when SC) and, when SC, T Diag(cs_v) into tile tt. Elements above the 8x8 block diagonal
// are not written (their zeros are set once by the caller). The fp32 blocks above the diagonal
// that the merges read are zeroed here when ZERO (sT shares memory with other data), else the
// caller keeps them zero. When SC and TT_LO, the bf16 rounding residue of T Diag(cs_v) is written
// too, into rows 64..127 of tile tt (so that hi + lo carries about 16 mantissa bits). Without EMIT
// no tile is written; instead the whole lower triangle of T (8x8 block diagonal included, zeros
// above the diagonal inside it) is left in sT in fp32, for the caller to convert. scr: 2048 floats
// of scratch.
// Not inlined: it gets its own register budget.
template <bool SC, int NW, bool ZERO = true, bool TT_LO = false, bool EMIT = true>
__device__ __noinline__ void unit_lower_inverse(const float* sL, float* sT, float* scr, uint8_t* tp, uint8_t* tt,
                                                const float* cs_c, const float* cs_v, int tid, int bar_id) {
  static_assert(NW >= 4 && NW <= 8, "warp count");
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  auto sync = [&] { group_sync(bar_id, 32 * NW); };
  constexpr uint32_t kLoRows = 64 * 128;  // byte offset of row 64 in a 64-column K-major tile
  auto emit1 = [&](int t, int i, float v) {
    if (!EMIT) return;
    const uint32_t off = canon(t, i, 128);
    *reinterpret_cast<__nv_bfloat16*>(tp + off) = __float2bfloat16_rn(SC ? v * cs_c[i] : v);
    if (SC) {
      const float x = v * cs_v[i];
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      *reinterpret_cast<__nv_bfloat16*>(tt + off) = hi;
      if (TT_LO) *reinterpret_cast<__nv_bfloat16*>(tt + kLoRows + off) = __float2bfloat16_rn(x - __bfloat162float(hi));
    }
  };
  auto emit2 = [&](int t, int i, float v0, float v1) {  // columns i, i + 1 (i even)
    if (!EMIT) return;
    const uint32_t off = canon(t, i, 128);
    *reinterpret_cast<uint32_t*>(tp + off) = pack_bf16(SC ? v0 * cs_c[i] : v0, SC ? v1 * cs_c[i + 1] : v1);
    if (SC && TT_LO) {
      uint32_t hi, lo;
      tc::split_bf16(v0 * cs_v[i], v1 * cs_v[i + 1], hi, lo);
      *reinterpret_cast<uint32_t*>(tt + off) = hi;
      *reinterpret_cast<uint32_t*>(tt + kLoRows + off) = lo;
    } else if (SC) {
      *reinterpret_cast<uint32_t*>(tt + off) = pack_bf16(v0 * cs_v[i], v1 * cs_v[i + 1]);
    }
  };
  if (tid < 64) {
    const int base = 8 * (tid >> 3), j = tid & 7;
    float x[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float s0 = (r == j) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
      for (int i = 0; i < r; ++i) {
        const float l = sL[xi(base + r, base + i)];
        if (i & 1)
          s1 = fmaf(-l, x[i], s1);
        else
          s0 = fmaf(-l, x[i], s0);
      }
      x[r] = s0 + s1;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      sT[xi(base + r, base + j)] = x[r];
      emit1(base + r, base + j, x[r]);
    }
  } else if (ZERO) {
    // zero, inside each 32x32 diagonal block, the 8x8 and 16x16 blocks above the diagonal that the
    // merge levels read: rows 16p..+8 x cols 16p+8..+8 (p < 4); rows 32q..+16 x cols 32q+16..+16 (q < 2)
    for (int e = tid - 64; e < 768; e += 32 * NW - 64) {
      if (e < 256) {
        const int p = e >> 6, r = (e >> 3) & 7, cc = e & 7;
        sT[xi(16 * p + r, 16 * p + 8 + cc)] = 0.f;
      } else {
        const int e2 = e - 256, q = e2 >> 8, r = (e2 >> 4) & 15, cc = e2 & 15;
        sT[xi(32 * q + r, 32 * q + 16 + cc)] = 0.f;
      }
    }
  }
  sync();
  // 8 -> 16: T_ba = -T_bb (L_ba T_aa) in each 16x16 diagonal block (rows 8..15 of the 16-row
  // mma operands repeat rows 0..7 and their results are ignored)
  if (warp < 4) {
    const int a0 = 16 * warp, b0 = a0 + 8;
    float* Y = scr + warp * 96;  // 8 x 12 (padded)
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<8>(d, [&](int i, int k) { return sL[xi(b0 + (i & 7), a0 + k)]; },
               [&](int k, int n) { return sT[xi(a0 + k, a0 + n)]; }, lane);
    Y[g * 12 + 2 * t4] = d[0];
    Y[g * 12 + 2 * t4 + 1] = d[1];
    __syncwarp();
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<8>(e, [&](int i, int k) { return sT[xi(b0 + (i & 7), b0 + k)]; },
               [&](int k, int n) { return Y[k * 12 + n]; }, lane);
    sT[xi(b0 + g, a0 + 2 * t4)] = -e[0];
    sT[xi(b0 + g, a0 + 2 * t4 + 1)] = -e[1];
    emit2(b0 + g, a0 + 2 * t4, -e[0], -e[1]);
  }
  sync();
  // 16 -> 32: T_{i,i-1} = -T_ii (L_{i,i-1} T_{i-1,i-1}) for (i, i-1) = (1, 0), (3, 2); warp w < 4
  // owns pair w / 2 and the 8-column tile w % 2 (a column tile of the result needs only the
  // same column tile of L T)
  if (warp < 4) {
    const int bi = 1 + 2 * (warp >> 1), bk = bi - 1, nt = warp & 1;
    float* Y = scr + 1152 + warp * 192;  // 16 x 12 (padded) dense scratch of this warp
    {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      warp_mm<16>(d, [&](int i, int k) { return sL[xi(16 * bi + i, 16 * bk + k)]; },
                  [&](int k, int n) { return sT[xi(16 * bk + k, 16 * bk + 8 * nt + n)]; }, lane);
      warp_store(d, [&](int i, int n, float v) { Y[i * 12 + n] = v; }, lane);
    }
    __syncwarp();
    {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      warp_mm<16>(d, [&](int i, int k) { return sT[xi(16 * bi + i, 16 * bi + k)]; },
                  [&](int k, int n) { return Y[k * 12 + n]; }, lane);
      warp_store2(d, [&](int i, int n, float v0, float v1) {
        sT[xi(16 * bi + i, 16 * bk + 8 * nt + n)] = -v0;
        sT[xi(16 * bi + i, 16 * bk + 8 * nt + n + 1)] = -v1;
        emit2(16 * bi + i, 16 * bk + 8 * nt + n, -v0, -v1);
      }, lane);
    }
  }
  sync();
  // 32 -> 64: X = L21 T1, then T21 = -T2 X; tile w covers rows 16 (w / 4) .. +16 and columns
  // 8 (w % 4) .. +8 of the 32x32 block; warp w owns tiles w, w + NW, ...
  float* X = scr;  // 32 x 36 (padded) dense
#pragma unroll
  for (int tile = warp; tile < 8; tile += NW) {
    const int mt = tile >> 2, nt = tile & 3;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<32>(d, [&](int i, int k) { return sL[xi(32 + 16 * mt + i, k)]; },
                [&](int k, int n) { return sT[xi(k, 8 * nt + n)]; }, lane);
    warp_store(d, [&](int i, int n, float v) { X[(16 * mt + i) * 36 + 8 * nt + n] = v; }, lane);
  }
  sync();
#pragma unroll
  for (int tile = warp; tile < 8; tile += NW) {
    const int mt = tile >> 2, nt = tile & 3;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<32>(d, [&](int i, int k) { return sT[xi(32 + 16 * mt + i, 32 + k)]; },
                [&](int k, int n) { return X[k * 36 + 8 * nt + n]; }, lane);
    warp_store2(d, [&](int i, int n, float v0, float v1) {
      if (!EMIT) {
        sT[xi(32 + 16 * mt + i, 8 * nt + n)] = -v0;
        sT[xi(32 + 16 * mt + i, 8 * nt + n + 1)] = -v1;
      }
      emit2(32 + 16 * mt + i, 8 * nt + n, -v0, -v1);
    }, lane);
  }
  sync();
}



}  // namespace ut
}  // namespace dn
