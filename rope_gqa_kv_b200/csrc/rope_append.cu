// rope_append.cu -- QK-RMSNorm + RoPE on q (in place) and on k, fused with the
// scatter of the rotated k and the raw v into the per-sequence KV cache.
//
// RoPE: page "750美元从零训练3个LLM：一位开发者的实战复盘", section "V1：现代架构基线";
// QK-norm: page "训练3.8B LLM至0.384 CORE，成本998美元 – Hugo Vergnes", section "设置";
// KV-cache append: first page, section "V3：扩容与推理优化".
//
// One CTA per token (b, t).  The CTA issues the loads of its first head vectors,
// then turns the token's position into the D/2 rotation angles (float64 angle
// p * base^(-2i/D) reduced to [-pi, pi] in float64, cos/sin in fp32) in shared
// memory, shared by all of the token's heads.  Each head vector
// is then owned by TPV threads: thread j holds the 16-byte chunk j of the first
// half (coordinates 8j..8j+7) and the matching chunk of the second half
// (coordinates D/2+8j..), i.e. exactly the 8 rotation pairs it needs, so every
// global access is a coalesced 16-byte vector and no data crosses threads except
// the RMSNorm sum of squares (an xor-shuffle within the TPV-lane group).
#include "common.cuh"

namespace gqa {

namespace {

constexpr int kThreads = 256;

template <int D>
struct RopeShape {
    static constexpr int kHalf = D / 2;
    static constexpr int kChunks = kHalf / 8;               // active lanes per vector
    static constexpr int kTPV = kChunks <= 4 ? 4 : 8;       // lanes per vector (pow2)
    static constexpr int kVecPerWarp = 32 / kTPV;
};

// Sum over the TPV-lane group (aligned, power of two) of this lane's value.
template <int TPV>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = TPV / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int D>
__device__ __forceinline__ void rotate_vector(const uint4 a_in, const uint4 b_in, uint4 &a_out,
                                              uint4 &b_out, const float *cs, const float *sn,
                                              int j, bool active, bool qk_norm, float eps) {
    using S = RopeShape<D>;
    float xa[8], xb[8];
    const uint32_t wa[4] = {a_in.x, a_in.y, a_in.z, a_in.w};
    const uint32_t wb[4] = {b_in.x, b_in.y, b_in.z, b_in.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        xa[2 * e] = bf16lo(wa[e]);
        xa[2 * e + 1] = bf16hi(wa[e]);
        xb[2 * e] = bf16lo(wb[e]);
        xb[2 * e + 1] = bf16hi(wb[e]);
    }
    if (qk_norm) {
        float ss = 0.f;
        if (active) {
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += xa[e] * xa[e] + xb[e] * xb[e];
        }
        ss = group_sum<S::kTPV>(ss);
        const float inv = rsqrtf(ss * (1.0f / D) + eps);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            xa[e] *= inv;
            xb[e] *= inv;
        }
    }
    uint32_t oa[4], ob[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float ya[2], yb[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = 8 * j + 2 * e + u;       // pair index
            const float c = active ? cs[i] : 0.f;
            const float s = active ? sn[i] : 0.f;
            const float a = xa[2 * e + u], b = xb[2 * e + u];
            ya[u] = a * c - b * s;
            yb[u] = a * s + b * c;
        }
        oa[e] = pack_bf16x2(ya[0], ya[1]);
        ob[e] = pack_bf16x2(yb[0], yb[1]);
    }
    a_out = make_uint4(oa[0], oa[1], oa[2], oa[3]);
    b_out = make_uint4(ob[0], ob[1], ob[2], ob[3]);
}

// Vectors of one token, in order: Hq query heads (if q), Hkv key heads and Hkv
// value heads (if k).  Query heads are rotated in place; key heads are rotated
// into the cache; value heads are copied into the cache bit for bit.
template <int D>
__global__ void __launch_bounds__(kThreads)
rope_append_kernel(uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const uint16_t *__restrict__ v, uint16_t *__restrict__ kc,
                   uint16_t *__restrict__ vc, const int32_t *__restrict__ pos0,
                   int32_t *__restrict__ new_len, int T, int Hq, int Hkv, int Lmax,
                   int qk_norm, float eps, float base, int32_t *status) {
    using S = RopeShape<D>;
    __shared__ float cs[S::kHalf];
    __shared__ float sn[S::kHalf];
    // A kernel launched after this one as a programmatic dependent (the prefill
    // or the decode) may start its prologue now; it waits for this grid to
    // complete before it reads anything written here.
    asm volatile("griddepcontrol.launch_dependents;");

    const int token = blockIdx.x;              // b * T + t
    const int b = token / T;
    const int t = token - b * T;
    const int p0 = pos0 ? pos0[b] : 0;
    const int p = p0 + t;

    bool write_cache = (k != nullptr);
    if (threadIdx.x == 0) {
        if (p0 < 0) {
            report(status, GQA_DEV_BAD_LEN);
        } else if (write_cache && p0 + T > Lmax) {
            report(status, GQA_DEV_CAPACITY);
        }
        if (new_len && t == 0) new_len[b] = p0 + T;
    }
    if (p0 < 0) return;
    if (write_cache && p0 + T > Lmax) write_cache = false;

    const int nq = q ? Hq : 0;
    const int nk = write_cache ? Hkv : 0;
    const int nvec = nq + 2 * nk;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int j = lane % S::kTPV;
    const int slot = lane / S::kTPV;
    const bool active = j < S::kChunks;
    constexpr int kSlots = (kThreads / 32) * S::kVecPerWarp;

    const size_t tok_q = (size_t)token * Hq * D;
    const size_t tok_kv = (size_t)token * Hkv * D;

    // Where vector vi comes from and goes to; `rotate` is false for value heads.
    auto locate = [&](int vi, const uint16_t *&src, uint16_t *&dst, bool &rotate) {
        if (vi < nq) {
            src = q + tok_q + (size_t)vi * D;
            dst = q + tok_q + (size_t)vi * D;
            rotate = true;
        } else if (vi < nq + nk) {
            const int h = vi - nq;
            src = k + tok_kv + (size_t)h * D;
            dst = kc + (((size_t)b * Hkv + h) * Lmax + p) * D;
            rotate = true;
        } else {
            const int h = min(vi - nq - nk, Hkv - 1);
            src = v + tok_kv + (size_t)h * D;
            dst = vc + (((size_t)b * Hkv + h) * Lmax + p) * D;
            rotate = false;
        }
    };

    // The first kPre passes of loads are issued before the angles are computed,
    // so their memory latency overlaps the trigonometry and the barrier.
    constexpr int kPre = 2;
    uint4 ra[kPre], rb[kPre];
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
        const int vi = u * kSlots + warp * S::kVecPerWarp + slot;
        ra[u] = make_uint4(0, 0, 0, 0);
        rb[u] = make_uint4(0, 0, 0, 0);
        if (vi < nvec && active) {
            const uint16_t *src;
            uint16_t *dst;
            bool rot;
            locate(vi, src, dst, rot);
            ra[u] = *reinterpret_cast<const uint4 *>(src + 8 * j);
            rb[u] = *reinterpret_cast<const uint4 *>(src + S::kHalf + 8 * j);
        }
    }

    // Angle p * base^(-2i/D) in float64, reduced to [-pi, pi] in float64
    // (subtracting the nearest multiple of 2*pi), then sin/cos in fp32.
    for (int i = threadIdx.x; i < S::kHalf; i += kThreads) {
        const double theta = pow((double)base, -2.0 * (double)i / (double)D);
        const double a = (double)p * theta;
        const double two_pi = 6.283185307179586476925286766559;
        const double r = a - rint(a * (1.0 / two_pi)) * two_pi;
        float sf, cf;
        sincosf((float)r, &sf, &cf);
        cs[i] = cf;
        sn[i] = sf;
    }
    __syncthreads();

    // Every lane of a group runs the loop the same number of times (the shuffle
    // in the norm needs the whole warp); inactive lanes just skip memory.
    for (int pass = 0; pass * kSlots < nvec; ++pass) {
        const int vi = pass * kSlots + warp * S::kVecPerWarp + slot;
        const bool live = vi < nvec;
        const uint16_t *src;
        uint16_t *dst;
        bool rotate;
        locate(live ? vi : 0, src, dst, rotate);
        const bool mem = live && active;
        uint4 a = make_uint4(0, 0, 0, 0), bb = make_uint4(0, 0, 0, 0);
        if (pass < kPre) {
#pragma unroll
            for (int u = 0; u < kPre; ++u)
                if (u == pass) {
                    a = ra[u];
                    bb = rb[u];
                }
        } else if (mem) {
            a = *reinterpret_cast<const uint4 *>(src + 8 * j);
            bb = *reinterpret_cast<const uint4 *>(src + S::kHalf + 8 * j);
        }
        // Every lane computes the rotation (the norm's shuffle spans the whole
        // warp); value vectors keep their loaded bits.
        uint4 oa, ob;
        rotate_vector<D>(a, bb, oa, ob, cs, sn, j, mem, qk_norm != 0, eps);
        if (rotate) {
            a = oa;
            bb = ob;
        }
        if (mem) {
            *reinterpret_cast<uint4 *>(dst + 8 * j) = a;
            *reinterpret_cast<uint4 *>(dst + S::kHalf + 8 * j) = bb;
        }
    }
}

template <int D>
cudaError_t launch(void *q, const void *k, const void *v, void *kc, void *vc,
                   const int32_t *pos0, int32_t *new_len, int B, int T, int Hq, int Hkv,
                   int Lmax, const gqa_rope_params &p, int32_t *status, cudaStream_t s) {
    const unsigned grid = (unsigned)B * (unsigned)T;
    rope_append_kernel<D><<<grid, kThreads, 0, s>>>(
        static_cast<uint16_t *>(q), static_cast<const uint16_t *>(k),
        static_cast<const uint16_t *>(v), static_cast<uint16_t *>(kc),
        static_cast<uint16_t *>(vc), pos0, new_len, T, Hq, Hkv, Lmax, p.qk_norm, p.eps,
        p.rope_base, status);
    return cudaGetLastError();
}

gqa_status dispatch(void *q, const void *k, const void *v, void *kc, void *vc,
                    const int32_t *pos0, int32_t *new_len, int B, int T, int Hq, int Hkv,
                    int D, int Lmax, const gqa_rope_params &p, int32_t *status,
                    void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch (D) {
        case 64: e = launch<64>(q, k, v, kc, vc, pos0, new_len, B, T, Hq, Hkv, Lmax, p, status, s); break;
        case 96: e = launch<96>(q, k, v, kc, vc, pos0, new_len, B, T, Hq, Hkv, Lmax, p, status, s); break;
        case 128: e = launch<128>(q, k, v, kc, vc, pos0, new_len, B, T, Hq, Hkv, Lmax, p, status, s); break;
        default: return GQA_ERR_UNSUPPORTED;
    }
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

bool params_ok(const gqa_rope_params &p) {
    return p.eps >= 0.f && p.rope_base > 1.f;
}

}  // namespace
}  // namespace gqa

using gqa_host::aligned16;
using gqa_host::head_dim_ok;

extern "C" gqa_status gqa_rope_apply(void *q, const int32_t *pos0, int B, int T, int H, int D,
                                     gqa_rope_params p, void *stream) {
    if (!q || B < 1 || T < 1 || H < 1 || !aligned16(q) || !gqa::params_ok(p))
        return GQA_ERR_INVALID_ARG;
    if (!head_dim_ok(D)) return GQA_ERR_UNSUPPORTED;
    if ((long long)B * T > 0x7fffffffLL) return GQA_ERR_INVALID_ARG;
    return gqa::dispatch(q, nullptr, nullptr, nullptr, nullptr, pos0, nullptr, B, T, H, 1, D,
                         128, p, nullptr, stream);
}

static gqa_status check_append(const void *k, const void *v, const void *kc, const void *vc,
                               int max_pos0_host, int B, int T, int Hkv, int D, int Lmax,
                               const gqa_rope_params &p) {
    if (!k || !v || !kc || !vc || B < 1 || T < 1 || Hkv < 1 || Lmax < 1)
        return GQA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(kc) || !aligned16(vc) || !gqa::params_ok(p))
        return GQA_ERR_INVALID_ARG;
    if (!head_dim_ok(D)) return GQA_ERR_UNSUPPORTED;
    if (Lmax % 128 != 0) return GQA_ERR_INVALID_ARG;
    if ((long long)B * T > 0x7fffffffLL) return GQA_ERR_INVALID_ARG;
    if (max_pos0_host >= 0 && (long long)max_pos0_host + T > Lmax) return GQA_ERR_CAPACITY;
    return GQA_OK;
}

extern "C" gqa_status kv_cache_append(const void *k, const void *v, void *k_cache, void *v_cache,
                                      const int32_t *pos0, int max_pos0_host, int32_t *new_len,
                                      int B, int T, int Hkv, int D, int Lmax, gqa_rope_params p,
                                      int32_t *status_dev, void *stream) {
    gqa_status st = check_append(k, v, k_cache, v_cache, max_pos0_host, B, T, Hkv, D, Lmax, p);
    if (st != GQA_OK) return st;
    return gqa::dispatch(nullptr, k, v, k_cache, v_cache, pos0, new_len, B, T, 1, Hkv, D, Lmax,
                         p, status_dev, stream);
}

extern "C" gqa_status gqa_rope_append(void *q, const void *k, const void *v, void *k_cache,
                                      void *v_cache, const int32_t *pos0, int max_pos0_host,
                                      int32_t *new_len, int B, int T, int Hq, int Hkv, int D,
                                      int Lmax, gqa_rope_params p, int32_t *status_dev,
                                      void *stream) {
    if (!q || Hq < 1 || Hkv < 1 || !aligned16(q)) return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    gqa_status st = check_append(k, v, k_cache, v_cache, max_pos0_host, B, T, Hkv, D, Lmax, p);
    if (st != GQA_OK) return st;
    return gqa::dispatch(q, k, v, k_cache, v_cache, pos0, new_len, B, T, Hq, Hkv, D, Lmax, p,
                         status_dev, stream);
}
