// fwht.cuh -- in-register Walsh-Hadamard butterflies shared by the row
// kernels (quant.cu: the DSFQ rotation; tq.cu: the 3DTurboQuant rotation).
// A row's values sit in a per-thread register array; a butterfly over index
// bit k combines entries j and j + 2^k into (sum, difference), the sum at the
// lower index (the Sylvester, natural-order Hadamard matrix).
//
// Row layout (one warp per row of K = 32*V values):
//   phase 1: lane l holds x[l + 32 j], j < V; the butterflies over the bits of
//            j (index bits 5 .. log2 K - 1) run in registers.
//   transpose through a 32 x 32 fp32 shared-memory tile per warp, V/32
//            passes: each lane writes its 32 values of a pass as one tile row
//            with 16-byte stores (16-byte chunk c of row l at chunk position
//            c ^ (l % 8): conflict-free both ways) and reads a column back.
//   phase 2: lane l holds x[V l + r], r < V: the butterflies over index bits
//            0..4 run in registers.
// For K = 1024 the two layouts are each other's transposes, so the same
// routine also takes a phase-2 row back to phase 1.
#pragma once

namespace w4a4 {
namespace {

// (a0, a1) <- (a0 + b0, a1 + b1), (b0, b1) <- (a0 - b0, a1 - b1) with the
// packed fp32x2 add/sub of sm_100 (each lane rounded exactly as a scalar add).
__device__ __forceinline__ void butterfly_x2(float &a0, float &a1, float &b0, float &b1) {
  unsigned long long A, B, S, D;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(S) : "l"(A), "l"(B));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(S));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(D));
}

// Butterflies for index bits [B0, B0 + NB) of a register array (natural order:
// the lower index of each pair receives the sum).  Distances >= 2 process two
// adjacent pairs per packed instruction.
template <int V, int B0, int NB>
__device__ __forceinline__ void butterflies(float (&v)[V]) {
#pragma unroll
  for (int s = 0; s < NB; ++s) {
    const int h = 1 << (B0 + s);
    if (h == 1) {
#pragma unroll
      for (int j = 0; j < V; j += 2) {
        const float a = v[j], b = v[j + 1];
        v[j] = a + b;
        v[j + 1] = a - b;
      }
    } else {
#pragma unroll
      for (int j = 0; j < V; j += 2)
        if ((j & h) == 0) butterfly_x2(v[j], v[j + 1], v[j + h], v[j + h + 1]);
    }
  }
}

// Register slot of phase-1 value j (x[lane + 32 j]).  The transpose pass
// p = j % (V/32) moves value j to lane j / (V/32); pass p writes tile column
// j / (V/32), and the four values of each 16-byte chunk of a pass sit in
// consecutive slots.  For K = 1024 (one pass) that is the identity; for
// K = 4096 the two low bits of j (the pass) and the next two swap places.
template <int K>
__host__ __device__ constexpr int phase1_slot(int j) {
  return K == 1024 ? j : (((j >> 2) & 3) | ((j & 3) << 2) | (j & ~15));
}

template <int K>
struct RowShape {
  static constexpr int V = K / 32;  // values per lane
  static constexpr int P = V / 32;  // transpose passes
  static constexpr int LOGV = (V == 32) ? 5 : 7;
  static constexpr float kInvSqrtK = (K == 1024) ? 0.03125f : 0.015625f;
  static_assert(K == 1024 || K == 4096, "K must be 1024 or 4096");
};

// Runs the transform (when ROT) on a phase-1 row u and leaves it in phase-2
// layout in v.
template <int K, bool ROT>
__device__ __forceinline__ void transform_row(float (&u)[RowShape<K>::V], int lane,
                                              float *__restrict__ tile, float (&v)[RowShape<K>::V]) {
  constexpr int V = RowShape<K>::V;
  constexpr int P = RowShape<K>::P;
  // index bits 5 .. log2(K)-1 (phase1_slot permutes them among themselves)
  if (ROT) butterflies<V, 0, RowShape<K>::LOGV>(u);
  float4 *trow = reinterpret_cast<float4 *>(tile + lane * 32);
#pragma unroll
  for (int p = 0; p < P; ++p) {
    // pass p: tile row `lane`, column c <- value j = P c + p of this lane
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int s0 = (K == 1024) ? 4 * m : 16 * m + 4 * p;
      trow[m ^ (lane & 7)] = make_float4(u[s0], u[s0 + 1], u[s0 + 2], u[s0 + 3]);
    }
    __syncwarp();
    // x[V lane + 32 p + l] is value j = P lane + p of lane l: column `lane` of row l
#pragma unroll
    for (int l = 0; l < 32; ++l)
      v[32 * p + l] = tile[l * 32 + ((((lane >> 2) ^ (l & 7)) << 2) | (lane & 3))];
    __syncwarp();
  }
  if (ROT) butterflies<V, 0, 5>(v);  // index bits 0..4
}

}  // namespace
}  // namespace w4a4
