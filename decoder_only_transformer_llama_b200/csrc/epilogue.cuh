// Fused projection epilogues (Admin Guide §8.4): rotary embedding of q and k
// plus the KV-cache append after wq/wk/wv, the residual add after wo and w2,
// silu(w1 x) * (w3 x) after the fused w1/w3 projection, and a plain fp32
// store for the vocabulary logits.
#pragma once

#include "common.cuh"
#include "model.h"

namespace llb {

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + __expf(-z)); }

// Rotate the adjacent pair (re, im) = (v[2j], v[2j+1]) by the angle of
// position `pos`, frequency j: (re*c - im*s, re*s + im*c).
__device__ __forceinline__ void rope_pair(const float2* rope, int hd, int pos, int j, float& re,
                                          float& im) {
    const float2 cs = rope[static_cast<long long>(pos) * (hd / 2) + j];
    const float a = re * cs.x - im * cs.y;
    const float b = re * cs.y + im * cs.x;
    re = a;
    im = b;
}

// QKV epilogue for one token row m and an even column pair (n, n+1) that
// lies inside one head.  Applies RoPE to q and k columns, writes q to the
// q buffer and k/v into the cache at (tok_row[m], head, tok_pos[m]).
template <typename T>
__device__ __forceinline__ void epi_qkv_pair(const Epi& ep, int m, int n, float v0, float v1) {
    const int pos = ep.tok_pos[m];
    if (pos < 0 || pos >= ep.max_seq) return;
    if (n < ep.nq) {
        const int d = n % ep.hd;
        rope_pair(ep.rope, ep.hd, pos, d >> 1, v0, v1);
        T* q = static_cast<T*>(ep.q) + static_cast<long long>(m) * ep.nq + n;
        q[0] = from_f32<T>(v0);
        q[1] = from_f32<T>(v1);
        return;
    }
    const int row = ep.tok_row ? ep.tok_row[m] : m;
    int c = n - ep.nq;
    T* cache = static_cast<T*>(ep.kc);
    const bool is_k = c < ep.nkvc;
    if (!is_k) {
        c -= ep.nkvc;
        cache = static_cast<T*>(ep.vc);
    }
    const int head = c / ep.hd, d = c % ep.hd;
    if (is_k) rope_pair(ep.rope, ep.hd, pos, d >> 1, v0, v1);
    T* dst = cache + static_cast<long long>(row) * ep.kv_row_stride +
             (static_cast<long long>(head) * ep.max_seq + pos) * ep.hd + d;
    dst[0] = from_f32<T>(v0);
    dst[1] = from_f32<T>(v1);
}

// Sum of x^2 of one token row from its n per-128-feature partial sums (fused
// RMSNorm, consumer side), added in order; the loads are issued eight at a
// time so that they are in flight together.
__device__ __forceinline__ float row_ssq(const float* p, int n) {
    float ss = 0.f;
    int t = 0;
    for (; t + 8 <= n; t += 8) {
        float a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) a[u] = p[t + u];
#pragma unroll
        for (int u = 0; u < 8; ++u) ss += a[u];
    }
    for (; t < n; ++t) ss += p[t];
    return ss;
}

}  // namespace llb
