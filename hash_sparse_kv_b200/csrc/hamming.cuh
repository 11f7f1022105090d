// Group-summed Hamming distance by bit-sliced arithmetic (HashEvict,
// "Abstract"; the GQA group sum of the retrieval kernels):
//     D(t) = sum_h popcount(cq_h XOR ck_t).
// For bit position j let c_j = #{h : bit j of cq_h is 1}; position j adds
// (ck_j ? g - c_j : c_j).  The NP bit planes of c_j (C) and of g - c_j (U)
// are built once per query group; per token each word gives NP planes
// V_b = (ck & U_b) | (~ck & C_b), words are added with ripple adders on the
// planes, and D = sum_b 2^b popcount(S_b).
#pragma once

#include <stdint.h>

namespace hkv {

template <int W, int NP>
struct Planes {
  uint32_t C[NP][W];
  uint32_t U[NP][W];
};

// Bit-sliced counters: C planes count the query codes' ones, U planes their zeros.
template <int W, int NP>
__device__ __forceinline__ void build_planes(const uint32_t* qc, int g, Planes<W, NP>& p) {
#pragma unroll
  for (int b = 0; b < NP; ++b)
#pragma unroll
    for (int w = 0; w < W; ++w) p.C[b][w] = p.U[b][w] = 0u;
  for (int h = 0; h < g; ++h) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const uint32_t q = qc[h * W + w];
      uint32_t carry = q;
#pragma unroll
      for (int b = 0; b < NP; ++b) {
        const uint32_t t = p.C[b][w] & carry;
        p.C[b][w] ^= carry;
        carry = t;
      }
      carry = ~q;
#pragma unroll
      for (int b = 0; b < NP; ++b) {
        const uint32_t t = p.U[b][w] & carry;
        p.U[b][w] ^= carry;
        carry = t;
      }
    }
  }
}

// s = a + b on bit-sliced numbers of NB planes (ripple of full adders).
template <int NB>
__device__ __forceinline__ void add_planes(const uint32_t (&a)[NB], const uint32_t (&b)[NB], uint32_t (&s)[NB + 1]) {
  uint32_t c = 0u;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const uint32_t x = a[i], y = b[i];
    s[i] = x ^ y ^ c;
    c = (x & y) | (c & (x ^ y));
  }
  s[NB] = c;
}

template <int L>
__device__ __forceinline__ int weighted_popc(const uint32_t (&s)[L]) {
  int r = 0;
#pragma unroll
  for (int b = 0; b < L; ++b) r += __popc(s[b]) << b;
  return r;
}

template <int W, int NP>
__device__ __forceinline__ int token_distance(const uint32_t (&ck)[W], const Planes<W, NP>& p) {
  uint32_t v[W][NP];
#pragma unroll
  for (int w = 0; w < W; ++w)
#pragma unroll
    for (int b = 0; b < NP; ++b) v[w][b] = (ck[w] & p.U[b][w]) | (~ck[w] & p.C[b][w]);
  if constexpr (W == 2) {
    uint32_t s[NP + 1];
    add_planes<NP>(v[0], v[1], s);
    return weighted_popc<NP + 1>(s);
  } else {
    static_assert(W == 4, "codes of 64 or 128 bits");
    uint32_t s01[NP + 1], s23[NP + 1], s[NP + 2];
    add_planes<NP>(v[0], v[1], s01);
    add_planes<NP>(v[2], v[3], s23);
    add_planes<NP + 1>(s01, s23, s);
    return weighted_popc<NP + 2>(s);
  }
}

}  // namespace hkv
