// rope_append.cu -- QK-RMSNorm + RoPE on q (in place) and on k, fused with the
// scatter of the rotated k and the raw v into the per-sequence KV cache.
//
// RoPE: page "750美元从零训练3个LLM：一位开发者的实战复盘", section "V1：现代架构基线";
// QK-norm: page "训练3.8B LLM至0.384 CORE，成本998美元 – Hugo Vergnes", section "设置";
// KV-cache append: first page, section "V3：扩容与推理优化".
//
// Prompts and chunks: one warp per token (rope_append_tok_kernel); decode, with
// its one token per sequence: one CTA per token (rope_append_kernel), so the
// batch's few tokens still spread over enough warps.  Either issues the loads
// of its first head vectors, then turns each token's position into the D/2
// rotation angles (float64 angle p * theta_i reduced to [-pi, pi] in float64,
// cos/sin in fp32) through shared memory, shared by all of the token's heads.
// The float64 table theta_i -- base^(-2i/D), or one of the
// context-extension variants (linear interpolation, NTK-aware, YaRN, see
// gqa.h) -- is computed once per call on the host and passed as a kernel
// parameter, together with YaRN's scale of the rotated vectors.  Each head vector
// is then owned by TPV threads: thread j holds the 16-byte chunk j of the first
// half (coordinates 8j..8j+7) and the matching chunk of the second half
// (coordinates D/2+8j..), i.e. exactly the 8 rotation pairs it needs, so every
// global access is a coalesced 16-byte vector and no data crosses threads except
// the RMSNorm sum of squares (an xor-shuffle within the TPV-lane group).
#include <cmath>

#include "common.cuh"

namespace gqa {

namespace {

constexpr int kThreads = 256;

// Rotation frequencies theta_i of the D/2 pairs (float64) and the factor the
// rotated vectors are multiplied by (1 except for YaRN).
struct RopeTable {
    double theta[64];
    float mscale;
};

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

// Two fp32 lanes at once (one issue slot each): d = a * b, d = a * b + c.
__device__ __forceinline__ void mul2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fma2(float &d0, float &d1, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// cos / sin (times the YaRN factor) of the 8 rotation pairs 8j .. 8j+7 that
// lane j of a vector group owns, read from a row of D/2 angles in shared memory;
// zero on lanes that own no pair.
template <int D>
__device__ __forceinline__ void lane_angles(const float *cs_row, const float *sn_row, int j,
                                            bool active, float (&c)[8], float (&sv)[8]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float4 cv = make_float4(0.f, 0.f, 0.f, 0.f), sq = cv;
        if (active) {
            cv = *reinterpret_cast<const float4 *>(cs_row + 8 * j + 4 * h);
            sq = *reinterpret_cast<const float4 *>(sn_row + 8 * j + 4 * h);
        }
        c[4 * h] = cv.x; c[4 * h + 1] = cv.y; c[4 * h + 2] = cv.z; c[4 * h + 3] = cv.w;
        sv[4 * h] = sq.x; sv[4 * h + 1] = sq.y; sv[4 * h + 2] = sq.z; sv[4 * h + 3] = sq.w;
    }
}

template <int D>
__device__ __forceinline__ void rotate_vector(const uint4 a_in, const uint4 b_in, uint4 &a_out,
                                              uint4 &b_out, const float (&c)[8],
                                              const float (&sv)[8], bool active, bool qk_norm,
                                              float eps) {
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
        // sum of squares and the scaling on coordinate pairs (packed f32x2)
        float s0 = 0.f, s1 = 0.f;
        if (active) {
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                fma2(s0, s1, xa[e], xa[e + 1], xa[e], xa[e + 1], s0, s1);
                fma2(s0, s1, xb[e], xb[e + 1], xb[e], xb[e + 1], s0, s1);
            }
        }
        const float ss = group_sum<S::kTPV>(s0 + s1);
        const float inv = rsqrtf(ss * (1.0f / D) + eps);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            mul2(xa[e], xa[e + 1], xa[e], xa[e + 1], inv, inv);
            mul2(xb[e], xb[e + 1], xb[e], xb[e + 1], inv, inv);
        }
    }
    // rotation of pairs (8j + 2e, 8j + 2e + 1) two at a time:
    //   ya = a c - b s,  yb = a s + b c
    uint32_t oa[4], ob[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float c0 = c[2 * e], c1 = c[2 * e + 1], s0 = sv[2 * e], s1 = sv[2 * e + 1];
        const float a0 = xa[2 * e], a1 = xa[2 * e + 1], b0 = xb[2 * e], b1 = xb[2 * e + 1];
        float ya0, ya1, yb0, yb1;
        mul2(ya0, ya1, b0, b1, -s0, -s1);
        fma2(ya0, ya1, a0, a1, c0, c1, ya0, ya1);
        mul2(yb0, yb1, b0, b1, c0, c1);
        fma2(yb0, yb1, a0, a1, s0, s1, yb0, yb1);
        oa[e] = pack_bf16x2(ya0, ya1);
        ob[e] = pack_bf16x2(yb0, yb1);
    }
    a_out = make_uint4(oa[0], oa[1], oa[2], oa[3]);
    b_out = make_uint4(ob[0], ob[1], ob[2], ob[3]);
}

// Vectors of one token, in order: Hq query heads (if q), Hkv key heads and Hkv
// value heads (if k).  Query heads are rotated in place; key heads are rotated
// into the cache; value heads are copied into the cache bit for bit.  This
// kernel's CTA takes TB consecutive tokens of one sequence (TB = 1: the decode
// step): its global loads go out in batches of kBatch passes (the first batch
// before the angles are computed), so every lane has several 32-byte loads in
// flight.
constexpr int kBatch = 4;

template <int D, int TB>
__global__ void __launch_bounds__(kThreads)
rope_append_kernel(uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                   const uint16_t *__restrict__ v, uint16_t *__restrict__ kc,
                   uint16_t *__restrict__ vc, const int32_t *__restrict__ pos0,
                   int32_t *__restrict__ new_len, int T, int Hq, int Hkv, int Lmax,
                   int qk_norm, float eps, const __grid_constant__ RopeTable tab,
                   int32_t *status) {
    using S = RopeShape<D>;
    __shared__ __align__(16) float cs[TB][S::kHalf];
    __shared__ __align__(16) float sn[TB][S::kHalf];
    // Launched as a programmatic dependent of whatever precedes it on the stream
    // (which may have produced q, k, v or pos0): wait for it before reading.  A
    // kernel launched after this one the same way (the prefill or the decode)
    // may then start its prologue; it waits for this grid to complete before it
    // reads anything written here.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    const int nblk = (T + TB - 1) / TB;
    const int b = blockIdx.x / nblk;
    const int t0 = (blockIdx.x - b * nblk) * TB;
    const int nt = min(TB, T - t0);
    const int p0 = pos0 ? pos0[b] : 0;

    bool write_cache = (k != nullptr);
    if (threadIdx.x == 0) {
        if (p0 < 0) {
            report(status, GQA_DEV_BAD_LEN);
        } else if (write_cache && p0 + T > Lmax) {
            report(status, GQA_DEV_CAPACITY);
        }
        if (new_len && t0 == 0) new_len[b] = p0 + T;
    }
    if (p0 < 0) return;
    if (write_cache && p0 + T > Lmax) write_cache = false;

    const int nq = q ? Hq : 0;
    const int nk = write_cache ? Hkv : 0;
    const int per_tok = nq + 2 * nk;
    const int nvec = nt * per_tok;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int j = lane % S::kTPV;
    const int slot = lane / S::kTPV;
    const bool active = j < S::kChunks;
    constexpr int kSlots = (kThreads / 32) * S::kVecPerWarp;
    const int npass = (nvec + kSlots - 1) / kSlots;

    // Where vector vi of the block comes from and goes to; `rotate` is false for
    // value heads, `tl` is its token within the block.
    auto locate = [&](int vi, const uint16_t *&src, uint16_t *&dst, bool &rotate, int &tl) {
        tl = vi / per_tok;
        const int r = vi - tl * per_tok;
        const int t = t0 + tl;
        const int p = p0 + t;
        const size_t token = (size_t)b * T + t;
        if (r < nq) {
            src = q + (token * Hq + r) * D;
            dst = q + (token * Hq + r) * D;
            rotate = true;
        } else if (r < nq + nk) {
            const int h = r - nq;
            src = k + (token * Hkv + h) * D;
            dst = kc + (((size_t)b * Hkv + h) * Lmax + p) * D;
            rotate = true;
        } else {
            const int h = r - nq - nk;
            src = v + (token * Hkv + h) * D;
            dst = vc + (((size_t)b * Hkv + h) * Lmax + p) * D;
            rotate = false;
        }
    };

    for (int pb = 0; pb < npass; pb += kBatch) {
        uint4 ra[kBatch], rb[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int vi = (pb + u) * kSlots + warp * S::kVecPerWarp + slot;
            ra[u] = make_uint4(0, 0, 0, 0);
            rb[u] = make_uint4(0, 0, 0, 0);
            if (vi < nvec && active) {
                const uint16_t *src;
                uint16_t *dst;
                bool rot;
                int tl;
                locate(vi, src, dst, rot, tl);
                ra[u] = *reinterpret_cast<const uint4 *>(src + 8 * j);
                rb[u] = *reinterpret_cast<const uint4 *>(src + S::kHalf + 8 * j);
            }
        }
        if (pb == 0) {
            // Angle p * theta_i in float64, reduced to [-pi, pi] in float64
            // (subtracting the nearest multiple of 2*pi), then sin/cos in fp32.
            for (int i = threadIdx.x; i < TB * S::kHalf; i += kThreads) {
                const int tl = i / S::kHalf, pi = i - tl * S::kHalf;
                const double a = (double)(p0 + t0 + tl) * tab.theta[pi];
                const double two_pi = 6.283185307179586476925286766559;
                const double r = a - rint(a * (1.0 / two_pi)) * two_pi;
                float sf, cf;
                sincosf((float)r, &sf, &cf);
                cs[tl][pi] = cf * tab.mscale;
                sn[tl][pi] = sf * tab.mscale;
            }
            __syncthreads();
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (pb + u >= npass) break;                    // uniform across the CTA
            const int vi = (pb + u) * kSlots + warp * S::kVecPerWarp + slot;
            const bool live = vi < nvec;
            const uint16_t *src;
            uint16_t *dst;
            bool rotate;
            int tl;
            locate(live ? vi : 0, src, dst, rotate, tl);
            const bool mem = live && active;
            // Every lane computes the rotation (the norm's shuffle spans the
            // whole warp); value vectors keep their loaded bits.
            uint4 a = ra[u], bb = rb[u], oa, ob;
            float c[8], sv[8];
            lane_angles<D>(cs[tl], sn[tl], j, mem, c, sv);
            rotate_vector<D>(a, bb, oa, ob, c, sv, mem, qk_norm != 0, eps);
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
}

// Prompts and chunks (T >= kTokWarps): one warp per token, kTokWarps tokens per
// CTA.  The warp walks its token's vectors -- Hq query heads, Hkv key heads, Hkv
// value heads -- kVecPerWarp at a time (one pass), loads kTokBatch passes ahead,
// and keeps the cos/sin of each lane's 8 pairs in registers for the whole token.
// A pass that holds value heads only skips the arithmetic.  Sources and
// destinations follow from the head index by adds alone.
constexpr int kTokWarps = 4;
constexpr int kTokBatch = 5;

template <int D>
__global__ void __launch_bounds__(kTokWarps * 32)
rope_append_tok_kernel(uint16_t *__restrict__ q, const uint16_t *__restrict__ k,
                       const uint16_t *__restrict__ v, uint16_t *__restrict__ kc,
                       uint16_t *__restrict__ vc, const int32_t *__restrict__ pos0,
                       int32_t *__restrict__ new_len, int T, int Hq, int Hkv, int Lmax,
                       int qk_norm, float eps, const __grid_constant__ RopeTable tab,
                       int32_t *status) {
    using S = RopeShape<D>;
    __shared__ __align__(16) float cs[kTokWarps][S::kHalf];
    __shared__ __align__(16) float sn[kTokWarps][S::kHalf];
    asm volatile("griddepcontrol.wait;" ::: "memory");     // as in rope_append_kernel
    asm volatile("griddepcontrol.launch_dependents;");

    const int nblk = (T + kTokWarps - 1) / kTokWarps;
    const int b = blockIdx.x / nblk;
    const int t0 = (blockIdx.x - b * nblk) * kTokWarps;
    const int p0 = pos0 ? pos0[b] : 0;

    bool write_cache = (k != nullptr);
    if (threadIdx.x == 0) {
        if (p0 < 0) {
            report(status, GQA_DEV_BAD_LEN);
        } else if (write_cache && p0 + T > Lmax) {
            report(status, GQA_DEV_CAPACITY);
        }
        if (new_len && t0 == 0) new_len[b] = p0 + T;
    }
    if (p0 < 0) return;
    if (write_cache && p0 + T > Lmax) write_cache = false;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t = t0 + warp;
    if (t >= T) return;                        // only warp-level sync follows
    const int p = p0 + t;
    const int j = lane % S::kTPV;
    const int slot = lane / S::kTPV;
    const bool active = j < S::kChunks;
    const int nq = q ? Hq : 0;
    const int nk = write_cache ? Hkv : 0;
    const int nrot = nq + nk;
    const int nvec = nrot + nk;
    const int npass = (nvec + S::kVecPerWarp - 1) / S::kVecPerWarp;
    const size_t token = (size_t)b * T + t;

    auto locate = [&](int r, const uint16_t *&src, uint16_t *&dst) {
        if (r < nq) {
            dst = q + (token * Hq + r) * D;
            src = dst;
        } else if (r < nrot) {
            const int h = r - nq;
            src = k + (token * Hkv + h) * D;
            dst = kc + (((size_t)b * Hkv + h) * Lmax + p) * D;
        } else {
            const int h = r - nrot;
            src = v + (token * Hkv + h) * D;
            dst = vc + (((size_t)b * Hkv + h) * Lmax + p) * D;
        }
    };

    float c[8], sv[8];
    for (int pb = 0; pb < npass; pb += kTokBatch) {
        uint4 ra[kTokBatch], rb[kTokBatch];
#pragma unroll
        for (int u = 0; u < kTokBatch; ++u) {
            const int r = (pb + u) * S::kVecPerWarp + slot;
            ra[u] = make_uint4(0, 0, 0, 0);
            rb[u] = make_uint4(0, 0, 0, 0);
            if (r < nvec && active) {
                const uint16_t *src;
                uint16_t *dst;
                locate(r, src, dst);
                ra[u] = *reinterpret_cast<const uint4 *>(src + 8 * j);
                rb[u] = *reinterpret_cast<const uint4 *>(src + S::kHalf + 8 * j);
            }
        }
        if (pb == 0) {
            // Angle p * theta_i in float64, reduced to [-pi, pi] in float64, then
            // sin/cos in fp32; the warp's row of D/2 angles goes through shared
            // memory to the lanes that own each pair.
            for (int i = lane; i < S::kHalf; i += 32) {
                const double a = (double)p * tab.theta[i];
                const double two_pi = 6.283185307179586476925286766559;
                const double r = a - rint(a * (1.0 / two_pi)) * two_pi;
                float sf, cf;
                sincosf((float)r, &sf, &cf);
                cs[warp][i] = cf * tab.mscale;
                sn[warp][i] = sf * tab.mscale;
            }
            __syncwarp();
            lane_angles<D>(cs[warp], sn[warp], j, active, c, sv);
        }
#pragma unroll
        for (int u = 0; u < kTokBatch; ++u) {
            if (pb + u >= npass) break;                    // uniform across the warp
            const int r0 = (pb + u) * S::kVecPerWarp;      // first vector of the pass
            const int r = r0 + slot;
            const bool mem = r < nvec && active;
            uint4 a = ra[u], bb = rb[u];
            if (r0 < nrot) {                               // uniform across the warp
                uint4 oa, ob;
                rotate_vector<D>(a, bb, oa, ob, c, sv, mem, qk_norm != 0, eps);
                if (r < nrot) {
                    a = oa;
                    bb = ob;
                }
            }
            if (mem) {
                const uint16_t *src;
                uint16_t *dst;
                locate(r, src, dst);
                *reinterpret_cast<uint4 *>(dst + 8 * j) = a;
                *reinterpret_cast<uint4 *>(dst + S::kHalf + 8 * j) = bb;
            }
        }
    }
}

// theta_i for the chosen variant, in float64 on the host (formulas in gqa.h).
RopeTable make_table(int D, const gqa_rope_params &p) {
    RopeTable t;
    const int half = D / 2;
    const double base = (double)p.rope_base, s = (double)p.factor;
    const double two_pi = 6.283185307179586476925286766559;
    double eff_base = base;
    if (p.scaling == GQA_ROPE_NTK) eff_base = base * std::pow(s, (double)D / (double)(D - 2));
    for (int i = 0; i < 64; ++i) t.theta[i] = 0.0;
    for (int i = 0; i < half; ++i) {
        const double th = std::pow(eff_base, -2.0 * (double)i / (double)D);
        double out = th;
        if (p.scaling == GQA_ROPE_LINEAR) {
            out = th / s;
        } else if (p.scaling == GQA_ROPE_YARN) {
            const double r = (double)p.original_max_pos * th / two_pi;
            double gmix = (r - (double)p.yarn_alpha) / ((double)p.yarn_beta - (double)p.yarn_alpha);
            gmix = gmix < 0.0 ? 0.0 : (gmix > 1.0 ? 1.0 : gmix);
            out = (1.0 - gmix) * th / s + gmix * th;
        }
        t.theta[i] = out;
    }
    t.mscale = p.scaling == GQA_ROPE_YARN ? (float)(0.1 * std::log(s) + 1.0) : 1.0f;
    return t;
}

// A launch as a programmatic dependent of the preceding kernel on the stream: its
// launch overlaps that kernel's last CTAs (the kernel waits for it on entry).
template <typename K, typename... Args>
cudaError_t launch_pdl(K kern, unsigned grid, unsigned block, cudaStream_t s, Args... args) {
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int D, int TB>
cudaError_t launch(void *q, const void *k, const void *v, void *kc, void *vc,
                   const int32_t *pos0, int32_t *new_len, int B, int T, int Hq, int Hkv,
                   int Lmax, const gqa_rope_params &p, int32_t *status, cudaStream_t s) {
    const unsigned grid = (unsigned)B * (unsigned)((T + TB - 1) / TB);
    return launch_pdl(rope_append_kernel<D, TB>, grid, kThreads, s, static_cast<uint16_t *>(q),
                      static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v),
                      static_cast<uint16_t *>(kc), static_cast<uint16_t *>(vc), pos0, new_len, T,
                      Hq, Hkv, Lmax, p.qk_norm, p.eps, make_table(D, p), status);
}

template <int D>
cudaError_t launch_tb(void *q, const void *k, const void *v, void *kc, void *vc,
                      const int32_t *pos0, int32_t *new_len, int B, int T, int Hq, int Hkv,
                      int Lmax, const gqa_rope_params &p, int32_t *status, cudaStream_t s) {
    // A warp per token once a sequence has kTokWarps tokens; otherwise (decode)
    // a whole CTA per token, so that the grid still spreads the batch's few
    // tokens over enough warps.
    if (T >= kTokWarps) {
        const unsigned grid = (unsigned)B * (unsigned)((T + kTokWarps - 1) / kTokWarps);
        return launch_pdl(rope_append_tok_kernel<D>, grid, kTokWarps * 32, s,
                          static_cast<uint16_t *>(q), static_cast<const uint16_t *>(k),
                          static_cast<const uint16_t *>(v), static_cast<uint16_t *>(kc),
                          static_cast<uint16_t *>(vc), pos0, new_len, T, Hq, Hkv, Lmax,
                          p.qk_norm, p.eps, make_table(D, p), status);
    }
    return launch<D, 1>(q, k, v, kc, vc, pos0, new_len, B, T, Hq, Hkv, Lmax, p, status, s);
}

gqa_status dispatch(void *q, const void *k, const void *v, void *kc, void *vc,
                    const int32_t *pos0, int32_t *new_len, int B, int T, int Hq, int Hkv,
                    int D, int Lmax, const gqa_rope_params &p, int32_t *status,
                    void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch (D) {
        case 64: e = launch_tb<64>(q, k, v, kc, vc, pos0, new_len, B, T, Hq, Hkv, Lmax, p, status, s); break;
        case 96: e = launch_tb<96>(q, k, v, kc, vc, pos0, new_len, B, T, Hq, Hkv, Lmax, p, status, s); break;
        case 128: e = launch_tb<128>(q, k, v, kc, vc, pos0, new_len, B, T, Hq, Hkv, Lmax, p, status, s); break;
        default: return GQA_ERR_UNSUPPORTED;
    }
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

bool params_ok(const gqa_rope_params &p) {
    if (!(p.eps >= 0.f && p.rope_base > 1.f)) return false;
    switch (p.scaling) {
        case GQA_ROPE_PLAIN: return true;
        case GQA_ROPE_LINEAR:
        case GQA_ROPE_NTK: return p.factor >= 1.f;
        case GQA_ROPE_YARN:
            return p.factor >= 1.f && p.original_max_pos >= 1 && p.yarn_alpha >= 0.f &&
                   p.yarn_beta > p.yarn_alpha;
        default: return false;
    }
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
