// Exact softmax attention over a query's leaf tokens with K/V rows loaded straight into
// registers (no shared-memory staging).  The final step of the decode path ("Subquadratic
// Attention with a Hierarchical Tree-Structured Indexer", abstract: attention runs over the
// sparse subset of keys the query's descent retrieved): every token of the query's leaves,
// softmax(q . k * scale) weights over those tokens, output sum_t w_t v_t.
//
// A token goes to LPT lanes (lane c = lane % LPT holds its 16-byte chunk c), TPP = 32 / LPT
// tokens per pass of a warp, PP passes per round with K and V of the round in flight
// together.  A warp keeps an online softmax in the log2 domain (scores are q . k times
// scale * log2 e): a warp-uniform running max, per-lane sums and output chunks.  One warp
// may take every token (slot 0 of 1), or several warps split them round by round (slot s
// of n takes rounds s, s + n, ...) and their states are merged afterwards.  K/V rows are
// read past L1 (each is read once).
#pragma once

#include "device_common.cuh"

namespace zha {

// 16 bytes from global memory through the non-coherent path, not kept in L1.
__device__ __forceinline__ uint4 ldg16_na(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float load_elem(const void* base, bool bf16, long long i) {
  return bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(base)[i]) : static_cast<const float*>(base)[i];
}

template <typename TKV, int D>
struct RegAttn {
  static constexpr int E = (int)sizeof(TKV);
  static constexpr int ROWB = D * E;       // bytes of a K or V row
  static constexpr int VEC = 16 / E;       // elements per 16-byte chunk
  static constexpr int LPT = ROWB / 16;    // lanes per token
  static constexpr int TPP = 32 / LPT;     // tokens per pass
  static_assert(LPT >= 1 && LPT <= 32 && 32 % LPT == 0, "row must split into 16-byte chunks over the warp");
};

// Tokens of the m leaves (ascending; only the last can be partial: the cache ends at N).
__device__ __forceinline__ int leaf_token_count(const int* leaves, int m, long long lb, long long N) {
  if (m <= 0) return 0;
  const long long last = leaves[m - 1];
  return (m - 1) * (int)lb + (int)(min(last * lb + lb, N) - last * lb);
}

// This lane's chunk of query qg (fp32).
template <typename TKV, int D>
__device__ __forceinline__ void reg_attn_load_q(const void* Q, bool q_bf16, long long qg, int lane,
                                                float (&qc)[RegAttn<TKV, D>::VEC]) {
  using A = RegAttn<TKV, D>;
  const int c = lane % A::LPT;
#pragma unroll
  for (int e = 0; e < A::VEC; ++e) qc[e] = load_elem(Q, q_bf16, qg * D + c * A::VEC + e);
}

// One warp's share of the tokens: rounds slot, slot + nslots, ... of TPP * PP tokens each.
// m_w (warp-uniform), l_w and acc (this lane's token group) carry the online softmax.
template <typename TKV, int D, int PP>
__device__ __forceinline__ void reg_attn_tokens(const int* leaves, int total, long long lb, const char* Ku,
                                                const char* Vu, const float (&qc)[RegAttn<TKV, D>::VEC],
                                                float qk_scale, int slot, int nslots, int lane, float& m_w,
                                                float& l_w, float (&acc)[RegAttn<TKV, D>::VEC]) {
  using A = RegAttn<TKV, D>;
  constexpr int VEC = A::VEC, LPT = A::LPT, TPP = A::TPP, ROWB = A::ROWB;
  const int c = lane % LPT, tg = lane / LPT;
  for (int s0 = slot * TPP * PP; s0 < total; s0 += nslots * TPP * PP) {
    uint4 kv[PP], vv[PP];
#pragma unroll
    for (int p = 0; p < PP; ++p) {
      const int s = s0 + p * TPP + tg;
      if (s < total) {
        const int j = s / (int)lb;
        const long long tok = (long long)leaves[j] * lb + (s - j * (int)lb);
        kv[p] = ldg16_na(Ku + tok * ROWB + c * 16);
        vv[p] = ldg16_na(Vu + tok * ROWB + c * 16);
      } else {
        kv[p] = make_uint4(0u, 0u, 0u, 0u);
        vv[p] = kv[p];
      }
    }
    float sc[PP];
    float mg = -INFINITY;
#pragma unroll
    for (int p = 0; p < PP; ++p) {
      float f[VEC];
      Vec16<TKV>::to_f32(kv[p], f);
      float2 d01 = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < VEC; e += 2)
        d01 = __ffma2_rn(make_float2(qc[e], qc[e + 1]), make_float2(f[e], f[e + 1]), d01);
      float d = d01.x + d01.y;
#pragma unroll
      for (int o = 1; o < LPT; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      sc[p] = s0 + p * TPP + tg < total ? d * qk_scale : -INFINITY;
      mg = fmaxf(mg, sc[p]);
    }
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, o));
    const float m_new = fmaxf(m_w, mg);
    const float alpha = m_w == -INFINITY ? 0.f : exp2f(m_w - m_new);
    l_w *= alpha;
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] *= alpha;
#pragma unroll
    for (int p = 0; p < PP; ++p) {
      const float pr = sc[p] == -INFINITY ? 0.f : exp2f(sc[p] - m_new);
      l_w += pr;
      float f[VEC];
      Vec16<TKV>::to_f32(vv[p], f);
#pragma unroll
      for (int e = 0; e < VEC; e += 2) {
        const float2 r = __ffma2_rn(make_float2(pr, pr), make_float2(f[e], f[e + 1]), make_float2(acc[e], acc[e + 1]));
        acc[e] = r.x;
        acc[e + 1] = r.y;
      }
    }
    m_w = m_new;
  }
}

// Sum the token groups' shares of l_w and of each output chunk (every lane ends with the
// warp's totals for its chunk c = lane % LPT).
template <typename TKV, int D>
__device__ __forceinline__ void reg_attn_fold(float& l_w, float (&acc)[RegAttn<TKV, D>::VEC]) {
  using A = RegAttn<TKV, D>;
#pragma unroll
  for (int o = A::LPT; o < 32; o <<= 1) {
    l_w += __shfl_xor_sync(0xffffffffu, l_w, o);
#pragma unroll
    for (int e = 0; e < A::VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  }
}

// Elements e0 .. e0 + N - 1 of output row qg: v[i] * inv, stored as bf16 or fp32.
template <int N>
__device__ __forceinline__ void store_out(void* O, bool o_bf16, long long qg, int D, int e0, const float (&v)[N],
                                          float inv) {
  if (o_bf16) {
    uint16_t* o16 = static_cast<uint16_t*>(O) + qg * D + e0;
#pragma unroll
    for (int e = 0; e < N; ++e) o16[e] = f32_to_bf16_bits(v[e] * inv);
  } else {
    float* o32 = static_cast<float*>(O) + qg * D + e0;
#pragma unroll
    for (int e = 0; e < N; ++e) o32[e] = v[e] * inv;
  }
}

}  // namespace zha
