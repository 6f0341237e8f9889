// Per-warp core of the exact decode attention ("Subquadratic Attention with a
// Hierarchical Tree-Structured Indexer", abstract: the final attention runs over the
// sparse subset of keys the tree traversal retrieved), shared by attend_kernel and the
// fused route + attention kernel.
//
//   s_t = scale * q . K[t],  o = sum_t exp(s_t - max) V[t] / sum_t exp(s_t - max)
//
// Layout of the work inside a warp: four lanes score one token from shared memory
// against q held in registers (lane (tg = lane / 4, sub = lane % 4) holds 16-byte chunks
// 4 (j ^ par) + sub of q, par = tg & 1, so the two tokens of a shared-memory phase read
// opposite bank halves); each lane accumulates head_dim / 32 output dims.  A warp keeps
// its own online softmax (running max and sum in the log2 domain) over the tokens it owns.
#pragma once

#include "device_common.cuh"

namespace zha {

template <typename TKV, int D>
struct AttnShape {
  static constexpr int E = sizeof(TKV);
  static constexpr int ROWB = D * E;      // bytes of one K or V row
  static constexpr int VEC = 16 / E;      // elements per 16-byte chunk
  static constexpr int NCH = ROWB / 16;   // 16-byte chunks per row
  static constexpr int CPL = NCH / 4;     // chunks per lane, four lanes per token
  static constexpr int DPL = D / 32;      // output dims per lane
  static_assert(NCH % 8 == 0, "row must split into an even number of chunks per lane");
};

// This lane's slice of query row qg (bf16 or fp32 storage) in the four-lanes-per-token
// chunk order of K dtype TKV.
template <typename TKV, int D>
__device__ __forceinline__ void attn_load_q(const void* Q, bool q_bf16, long long qg, int lane,
                                            float (&qv)[AttnShape<TKV, D>::CPL][AttnShape<TKV, D>::VEC]) {
  using S = AttnShape<TKV, D>;
  const int sub = lane & 3, par = (lane >> 2) & 1;
  const unsigned char* qrow = static_cast<const unsigned char*>(Q) + qg * D * (q_bf16 ? 2 : 4);
  if (q_bf16) {
#pragma unroll
    for (int j = 0; j < S::CPL; ++j) {
      const int c = 4 * (j ^ par) + sub;
      if constexpr (S::VEC == 8) {  // bf16 K: a chunk is 16 bytes of q as well
        float f[8];
        Vec16<uint16_t>::to_f32(ldg16(qrow + (size_t)c * 16), f);
#pragma unroll
        for (int k = 0; k < 8; ++k) qv[j][k] = f[k];
      } else {  // fp32 K: four bf16 elements, 8 bytes (8-byte aligned only)
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(qrow + (size_t)c * 8));
        qv[j][0] = bf16_bits_to_f32(v.x & 0xFFFFu);
        qv[j][1] = bf16_bits_to_f32(v.x >> 16);
        qv[j][2] = bf16_bits_to_f32(v.y & 0xFFFFu);
        qv[j][3] = bf16_bits_to_f32(v.y >> 16);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < S::CPL; ++j) {
      const int c = 4 * (j ^ par) + sub;
#pragma unroll
      for (int e = 0; e < S::VEC; e += 4) {
        const uint4 v = ldg16(qrow + (size_t)(c * S::VEC + e) * 4);
        float f[4];
        Vec16<float>::to_f32(v, f);
#pragma unroll
        for (int k = 0; k < 4 && e + k < S::VEC; ++k) qv[j][e + k] = f[k];
      }
    }
  }
}

template <int D>
__device__ __forceinline__ void attn_load_v(const uint16_t* p, float* o) {
  if constexpr (D / 32 == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    o[0] = __uint_as_float(v.x << 16);
    o[1] = __uint_as_float(v.x & 0xFFFF0000u);
    o[2] = __uint_as_float(v.y << 16);
    o[3] = __uint_as_float(v.y & 0xFFFF0000u);
  } else {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
    o[0] = __uint_as_float(v << 16);
    o[1] = __uint_as_float(v & 0xFFFF0000u);
  }
}
template <int D>
__device__ __forceinline__ void attn_load_v(const float* p, float* o) {
  if constexpr (D / 32 == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x;
    o[1] = v.y;
    o[2] = v.z;
    o[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(p);
    o[0] = v.x;
    o[1] = v.y;
  }
}

// One warp's share of a staged run of cnt tokens (K rows at Ks, V rows at Vs, row-major):
// rounds of 16 tokens t0 + tg and t0 + off + tg for t0 = first, first + step, ...
// (off >= 8, step >= off + 8, so no token is taken twice).  Updates the warp's softmax
// state (m_w: running max, log2 domain, warp-uniform; l_w: this lane's part of the running
// sum; acc: this lane's output dims).  pw: 16 floats of shared memory private to the warp.
template <typename TKV, int D>
__device__ __forceinline__ void attn_tokens(const unsigned char* Ks, const unsigned char* Vs, int cnt,
                                            int first, int off, int step,
                                            const float (&qv)[AttnShape<TKV, D>::CPL][AttnShape<TKV, D>::VEC],
                                            float qk_scale, float* pw, float& m_w, float& l_w,
                                            float (&acc)[AttnShape<TKV, D>::DPL], int lane) {
  using S = AttnShape<TKV, D>;
  const int sub = lane & 3, tg = lane >> 2, par = tg & 1;
  for (int t0 = first; t0 < cnt; t0 += step) {
    float sc[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int t = t0 + off * u + tg;
      float2 d01 = make_float2(0.f, 0.f);  // even / odd dims, updated by packed FMAs
      if (t < cnt) {
        const unsigned char* row = Ks + (size_t)t * S::ROWB;
#pragma unroll
        for (int j = 0; j < S::CPL; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(row + (4 * (j ^ par) + sub) * 16);
          float f[S::VEC];
          Vec16<TKV>::to_f32(v, f);
#pragma unroll
          for (int e = 0; e < S::VEC; e += 2)
            d01 = __ffma2_rn(make_float2(qv[j][e], qv[j][e + 1]), make_float2(f[e], f[e + 1]), d01);
        }
      }
      float d = d01.x + d01.y;
      d += __shfl_xor_sync(0xffffffffu, d, 1);
      d += __shfl_xor_sync(0xffffffffu, d, 2);
      sc[u] = t < cnt ? d * qk_scale : -INFINITY;
    }
    float mg = fmaxf(sc[0], sc[1]);
    mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, 4));
    mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, 8));
    mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, 16));
    const float m_new = fmaxf(m_w, mg);
    const float alpha = m_w == -INFINITY ? 0.f : exp2f(m_w - m_new);
    const float p0 = sc[0] == -INFINITY ? 0.f : exp2f(sc[0] - m_new);
    const float p1 = sc[1] == -INFINITY ? 0.f : exp2f(sc[1] - m_new);
    l_w = l_w * alpha + (sub == 0 ? p0 + p1 : 0.f);  // per lane; summed over the warp at the end
    m_w = m_new;
    if (sub == 0) {
      pw[tg] = p0;
      pw[8 + tg] = p1;
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < S::DPL; ++e) acc[e] *= alpha;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = t0 + (j < 8 ? j : off + j - 8);  // tokens t0 .. t0+7 and t0+off .. t0+off+7
      if (t < cnt) {
        const float p = pw[j];
        float v[S::DPL];
        attn_load_v<D>(reinterpret_cast<const TKV*>(Vs + (size_t)t * S::ROWB) + lane * S::DPL, v);
#pragma unroll
        for (int e = 0; e < S::DPL; e += 2) {
          const float2 r = __ffma2_rn(make_float2(p, p), make_float2(v[e], v[e + 1]),
                                      make_float2(acc[e], acc[e + 1]));
          acc[e] = r.x;
          acc[e + 1] = r.y;
        }
      }
    }
    __syncwarp();
  }
}

}  // namespace zha
