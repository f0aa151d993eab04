// decode.cu -- single-token attention against the KV cache (split-K, HBM-bound).
//
// One query token per sequence attends over lens[b] cached keys: the KV-cache
// step of page "750美元从零训练3个LLM：一位开发者的实战复盘", section
// "V3：扩容与推理优化" (per-step cost O(n) instead of O(n^2)), batched as on page
// "从零手训LLaMa：125M模型11小时训练全记录"; the cache is read once per GQA group,
// never once per query head (first page, section "V2：引入前沿技术").
//
// Work split: CTA (split, kv-head [x head subgroup], b) owns CH consecutive cache
// slots of one KV head and G of its query heads.  One thread issues two bulk
// copies (the K chunk and the V chunk, each one contiguous [n, D] block of the
// per-head slab) into shared memory; the four warps then
//   1. score: 4 lanes per key, each lane D/4 coordinates held against G query
//      vectors kept in registers; two xor-shuffles finish each dot product.
//      Lanes visit their 16-byte chunks in a rotated order (and the query
//      registers were loaded in that same order) so the 8 lanes of each
//      shared-memory phase hit 8 different bank groups.
//   2. chunk softmax in base 2: m = max, p = 2^(s - m), l = sum p.
//   3. p.V: lane (key group, 16-byte column chunk) accumulates G x 8 outputs
//      over its keys, then the key groups are summed through shared memory.
// The partial (m, l, o) of each split goes to the workspace; a second kernel,
// launched as a programmatic dependent of the first, merges the splits of each
// (b, query head): M = max m_i, o = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i.
#include "common.cuh"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int kDecThreads = 128;

template <int D, int G, int CH>
struct DecShape {
    static constexpr int kLaneChunks = D / 32;                  // 16-byte chunks per lane (score)
    static constexpr int kPasses = CH / 32;                     // 32 keys per pass
    static constexpr int kColChunks = D / 8;                    // 16-byte chunks per row (p.V)
    static constexpr int kKeyGroups = kDecThreads / kColChunks; // p.V key groups
    static constexpr int kKBytes = CH * D * 2;
    static constexpr int kPartialBytes = kKeyGroups * G * D * 4;
    static constexpr bool kAliasPartial = kPartialBytes <= kKBytes;
    // layout: [K chunk][V chunk][p: G x CH f32][red: 2 x 4 x G f32][partial (if not aliased)]
    static constexpr int kOffV = kKBytes;
    static constexpr int kOffP = 2 * kKBytes;
    static constexpr int kOffRed = kOffP + G * CH * 4;
    static constexpr int kOffPartial = kAliasPartial ? 0 : kOffRed + 2 * 4 * G * 4;
    static constexpr int kSmem = (kAliasPartial ? kOffRed + 2 * 4 * G * 4
                                                : kOffPartial + kPartialBytes) + 16;
};

// Rotation of a lane's chunk order that keeps each 8-lane phase conflict free.
template <int D>
__device__ __forceinline__ int chunk_rot(int lane) {
    const int j = lane & 3, kl = (lane >> 2) & 1;
    if (D == 128) return (j >> 1) + 2 * kl;
    if (D == 64) return kl;
    return 0;
}

template <int D, int G, int CH>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ kc,
                    const uint16_t *__restrict__ vc, const int32_t *__restrict__ lens,
                    int max_len, int Hq, int Hkv, int Lmax, float scale_log2, int n_splits,
                    int n_sub, float *__restrict__ ws_o, float *__restrict__ ws_ml,
                    int32_t *status) {
    using S = DecShape<D, G, CH>;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[2];

    // The merge kernel may be scheduled now; it waits for this grid to finish
    // before it reads anything.
    asm volatile("griddepcontrol.launch_dependents;");
    const int split = blockIdx.x;
    const int kvh = blockIdx.y / n_sub;
    const int sub = blockIdx.y - kvh * n_sub;
    const int b = blockIdx.z;
    const int tid = threadIdx.x;
    const int len = lens[b];
    if (len < 1 || len > max_len || len > Lmax) {
        if (split == 0 && blockIdx.y == 0 && tid == 0)
            report(status, len < 1 ? GQA_DEV_BAD_LEN : GQA_DEV_CAPACITY);
        return;
    }
    const int key0 = split * CH;
    if (key0 >= len) return;
    const int n = min(CH, len - key0);
    const int g = Hq / Hkv;
    const int h0 = kvh * g + sub * G;        // first query head of this CTA

    const uint32_t bar_k = ptx::smem_addr(&bars[0]);
    const uint32_t bar_v = ptx::smem_addr(&bars[1]);
    const uint16_t *ks = reinterpret_cast<const uint16_t *>(smem);
    const uint16_t *vs = reinterpret_cast<const uint16_t *>(smem + S::kOffV);
    float *ps = reinterpret_cast<float *>(smem + S::kOffP);
    float *red = reinterpret_cast<float *>(smem + S::kOffRed);
    float *partial = reinterpret_cast<float *>(smem + S::kOffPartial);

    if (tid == 0) {
        ptx::mbar_init(bar_k, 1);
        ptx::mbar_init(bar_v, 1);
        ptx::fence_barrier_init();
        const size_t slab = ((size_t)b * Hkv + kvh) * Lmax + key0;
        const uint32_t bytes = (uint32_t)n * D * 2;
        const uint64_t pol = ptx::policy_evict_first();
        ptx::mbar_arrive_expect_tx(bar_k, bytes);
        ptx::bulk_g2s_hint(ptx::smem_addr(smem), kc + slab * D, bytes, bar_k, pol);
        ptx::mbar_arrive_expect_tx(bar_v, bytes);
        ptx::bulk_g2s_hint(ptx::smem_addr(smem + S::kOffV), vc + slab * D, bytes, bar_v, pol);
    }

    // Query registers, in this lane's rotated chunk order (overlaps the copies).
    const int lane = tid & 31, warp = tid >> 5;
    const int j = lane & 3;
    const int rot = chunk_rot<D>(lane);
    float qr[G][S::kLaneChunks][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const uint16_t *qh = q + ((size_t)b * Hq + h0 + h) * D + j * (D / 4);
#pragma unroll
        for (int i = 0; i < S::kLaneChunks; ++i) {
            const int c = (i + rot) % S::kLaneChunks;
            const uint4 w = *reinterpret_cast<const uint4 *>(qh + c * 8);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                qr[h][i][2 * e] = bf16lo(ww[e]);
                qr[h][i][2 * e + 1] = bf16hi(ww[e]);
            }
        }
    }
    __syncthreads();   // barrier init visible to all threads

    bool ok = ptx::mbar_wait(bar_k, 0);
    // ---- 1. scores ------------------------------------------------------------
#pragma unroll
    for (int pass = 0; pass < S::kPasses; ++pass) {
        const int key = pass * 32 + warp * 8 + (lane >> 2);
        const uint16_t *krow = ks + key * D + j * (D / 4);
        float acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
        for (int i = 0; i < S::kLaneChunks; ++i) {
            const int c = (i + rot) % S::kLaneChunks;
            const uint4 w = *reinterpret_cast<const uint4 *>(krow + c * 8);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float k0 = bf16lo(ww[e]), k1 = bf16hi(ww[e]);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    acc[h] = fmaf(qr[h][i][2 * e], k0, acc[h]);
                    acc[h] = fmaf(qr[h][i][2 * e + 1], k1, acc[h]);
                }
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 1);
            acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], 2);
        }
        if (j == 0) {
#pragma unroll
            for (int h = 0; h < G; ++h)
                ps[h * CH + key] = key < n ? acc[h] * scale_log2 : -INFINITY;
        }
    }
    __syncthreads();

    // ---- 2. chunk softmax (base 2) --------------------------------------------
    float m[G], l[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float s = -INFINITY;
        for (int key = tid; key < CH; key += kDecThreads) s = fmaxf(s, ps[h * CH + key]);
        s = warp_max(s);
        if (lane == 0) red[warp * G + h] = s;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = fmaxf(fmaxf(red[0 * G + h], red[1 * G + h]), fmaxf(red[2 * G + h], red[3 * G + h]));
        float sum = 0.f;
        for (int key = tid; key < CH; key += kDecThreads) {
            const float p = ex2(ps[h * CH + key] - m[h]);
            ps[h * CH + key] = p;
            sum += p;
        }
        sum = warp_sum(sum);
        if (lane == 0) red[4 * G + warp * G + h] = sum;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h)
        l[h] = (red[4 * G + 0 * G + h] + red[4 * G + 1 * G + h]) +
               (red[4 * G + 2 * G + h] + red[4 * G + 3 * G + h]);

    // ---- 3. p . V ---------------------------------------------------------------
    ok = ptx::mbar_wait(bar_v, 0) && ok;
    const int col = tid % S::kColChunks;
    const int kg = tid / S::kColChunks;
    float o[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = 0.f;
    if (kg < S::kKeyGroups) {
        for (int key = kg; key < n; key += S::kKeyGroups) {
            const uint4 w = *reinterpret_cast<const uint4 *>(vs + key * D + col * 8);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            float pv[G];
#pragma unroll
            for (int h = 0; h < G; ++h) pv[h] = ps[h * CH + key];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float v0 = bf16lo(ww[e]), v1 = bf16hi(ww[e]);
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    o[h][2 * e] = fmaf(pv[h], v0, o[h][2 * e]);
                    o[h][2 * e + 1] = fmaf(pv[h], v1, o[h][2 * e + 1]);
                }
            }
        }
    }
    if (S::kAliasPartial) __syncthreads();   // every lane is done reading K
    if (kg < S::kKeyGroups) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float4 *dst = reinterpret_cast<float4 *>(partial + (kg * G + h) * D + col * 8);
            dst[0] = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
            dst[1] = make_float4(o[h][4], o[h][5], o[h][6], o[h][7]);
        }
    }
    __syncthreads();
    const size_t row0 = ((size_t)b * Hq + h0) * n_splits + split;   // (b, h0, split)
    for (int idx = tid; idx < G * D; idx += kDecThreads) {
        const int h = idx / D, d = idx - h * D;
        float acc = 0.f;
#pragma unroll 4
        for (int gi = 0; gi < S::kKeyGroups; ++gi) acc += partial[(gi * G + h) * D + d];
        ws_o[(row0 + (size_t)h * n_splits) * D + d] = acc;
    }
    if (tid < G) {
        float mm = 0.f, ll = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h)
            if (h == tid) { mm = m[h]; ll = l[h]; }
        ws_ml[(row0 + (size_t)tid * n_splits) * 2 + 0] = mm;
        ws_ml[(row0 + (size_t)tid * n_splits) * 2 + 1] = ll;
    }
    if (!ok) {
        // A copy that missed its deadline may still land in this CTA's shared
        // memory: give both one more bounded wait before the CTA retires.
        ptx::mbar_wait(bar_k, 0);
        ptx::mbar_wait(bar_v, 0);
        if (tid == 0) report(status, GQA_DEV_TIMEOUT);
    }
}

// Merge the splits of one (b, query head): one warp per row.  Lanes read the
// splits' (m, l) in parallel and reduce them with shuffles; each lane then owns
// D/32 output coordinates and walks the splits with independent loads.
constexpr int kCombWarps = 8;

template <int D>
__global__ void __launch_bounds__(kCombWarps * 32)
decode_combine_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_ml,
                      const int32_t *__restrict__ lens, int max_len, int B, int Hq, int Lmax,
                      int n_splits, int CH, uint16_t *__restrict__ out) {
    // Programmatic dependent launch: everything above this line may overlap the
    // split kernel; the partials are read only after it has completed.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kCombWarps + (threadIdx.x >> 5);   // b * Hq + h
    if (row >= B * Hq) return;
    const int b = row / Hq;
    const int len = lens[b];
    constexpr int kPer = D / 32;
    uint16_t *o = out + (size_t)row * D;
    if (len < 1 || len > max_len || len > Lmax) {
#pragma unroll
        for (int k = 0; k < kPer; ++k) o[lane + 32 * k] = 0;
        return;
    }
    const int ns = (len + CH - 1) / CH;
    const float *ml = ws_ml + (size_t)row * n_splits * 2;
    const float *po = ws_o + (size_t)row * n_splits * D;
    float M = -INFINITY;
    for (int i = lane; i < ns; i += 32) M = fmaxf(M, ml[2 * i]);
    M = warp_max(M);
    float L = 0.f;
    for (int i = lane; i < ns; i += 32) L = fmaf(ex2(ml[2 * i] - M), ml[2 * i + 1], L);
    L = warp_sum(L);
    float acc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
#pragma unroll 4
    for (int i = 0; i < ns; ++i) {
        const float w = ex2(ml[2 * i] - M);
#pragma unroll
        for (int k = 0; k < kPer; ++k) acc[k] = fmaf(w, po[(size_t)i * D + lane + 32 * k], acc[k]);
    }
    const float inv = 1.f / L;
#pragma unroll
    for (int k = 0; k < kPer; ++k)
        o[lane + 32 * k] = (uint16_t)(pack_bf16x2(acc[k] * inv, 0.f) & 0xffffu);
}

template <int D, int G, int CH>
cudaError_t launch_decode(const void *q, const void *kc, const void *vc, const int32_t *lens,
                          int max_len, void *out, int B, int Hq, int Hkv, int Lmax,
                          float scale_log2, float *ws_o, float *ws_ml, int n_splits,
                          int32_t *status, cudaStream_t s) {
    using S = DecShape<D, G, CH>;
    auto kern = decode_split_kernel<D, G, CH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::kSmem);
    if (e != cudaSuccess) return e;
    const int n_sub = (Hq / Hkv) / G;
    dim3 grid(n_splits, Hkv * n_sub, B);
    kern<<<grid, kDecThreads, S::kSmem, s>>>(
        static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(kc),
        static_cast<const uint16_t *>(vc), lens, max_len, Hq, Hkv, Lmax, scale_log2, n_splits,
        n_sub, ws_o, ws_ml, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // The merge is launched as a programmatic dependent of the split kernel, so
    // its launch and scheduling overlap the split kernel's last wave.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((B * Hq + kCombWarps - 1) / kCombWarps));
    cfg.blockDim = dim3(kCombWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, (const float *)ws_o,
                              (const float *)ws_ml, lens, max_len, B, Hq, Lmax, n_splits, CH,
                              static_cast<uint16_t *>(out));
}

// Query heads per CTA: the largest of {3, 2, 1} (D = 128) or {4, 3, 2, 1}
// dividing the group size g, bounded by the registers the query vectors take.
int heads_per_cta(int g, int D) {
    const int cap = D == 128 ? 3 : 4;
    for (int G = cap; G > 1; --G)
        if (g % G == 0) return G;
    return 1;
}

template <int D, int CH>
cudaError_t launch_g(int G, const void *q, const void *kc, const void *vc, const int32_t *lens,
                     int max_len, void *out, int B, int Hq, int Hkv, int Lmax, float sl2,
                     float *wo, float *wml, int ns, int32_t *st, cudaStream_t s) {
    switch (G) {
        case 1: return launch_decode<D, 1, CH>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, wo, wml, ns, st, s);
        case 2: return launch_decode<D, 2, CH>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, wo, wml, ns, st, s);
        case 3: return launch_decode<D, 3, CH>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, wo, wml, ns, st, s);
        default:
            if constexpr (D != 128)
                return launch_decode<D, 4, CH>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, wo, wml, ns, st, s);
            return cudaErrorInvalidValue;
    }
}

constexpr int kMinSplitChunk = 64;

// Chunk length: 128 slots when that still yields about two CTAs per SM,
// otherwise 64 (short caches / small batches are latency-bound).
int pick_chunk(int B, int Hkv, int n_sub, int max_len) {
    const long long ctas128 = (long long)B * Hkv * n_sub * ((max_len + 127) / 128);
    return ctas128 >= 2 * 148 ? 128 : 64;
}

}  // namespace
}  // namespace gqa

extern "C" size_t gqa_decode_workspace_bytes(int B, int Hq, int D, int max_len) {
    if (B < 1 || Hq < 1 || max_len < 1 || !gqa_host::head_dim_ok(D)) return 0;
    const size_t ns = (size_t)(max_len + gqa::kMinSplitChunk - 1) / gqa::kMinSplitChunk;
    const size_t rows = (size_t)B * Hq * ns;
    return rows * (size_t)D * 4 + rows * 2 * 4 + 256;
}

extern "C" gqa_status gqa_decode(const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *lens, int max_len_host, void *out, int B, int Hq,
                                 int Hkv, int D, int Lmax, float scale, void *ws, size_t ws_bytes,
                                 int32_t *status_dev, void *stream) {
    using namespace gqa_host;
    if (!q || !k_cache || !v_cache || !lens || !out || B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1)
        return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || B > 65535 || Hq > 65535) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(lens) & 3u))
        return GQA_ERR_INVALID_ARG;
    if (!head_dim_ok(D)) return GQA_ERR_UNSUPPORTED;
    if (Lmax % 128 != 0) return GQA_ERR_INVALID_ARG;
    if (max_len_host < 1) return GQA_ERR_INVALID_ARG;
    if (max_len_host > Lmax) return GQA_ERR_CAPACITY;
    const size_t need = gqa_decode_workspace_bytes(B, Hq, D, max_len_host);
    if (!ws || ws_bytes < need || !aligned16(ws)) return GQA_ERR_WORKSPACE;

    const int g = Hq / Hkv;
    const int G = gqa::heads_per_cta(g, D);
    const int CH = gqa::pick_chunk(B, Hkv, g / G, max_len_host);
    const int ns = (max_len_host + CH - 1) / CH;
    const size_t rows = (size_t)B * Hq * ns;
    float *ws_o = static_cast<float *>(ws);
    float *ws_ml = ws_o + rows * D;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
    const float sl2 = sc * 1.4426950408889634f;   // scores in base-2 units
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (CH == 128) {
        switch (D) {
            case 64: e = gqa::launch_g<64, 128>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws_o, ws_ml, ns, status_dev, s); break;
            case 96: e = gqa::launch_g<96, 128>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws_o, ws_ml, ns, status_dev, s); break;
            default: e = gqa::launch_g<128, 128>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws_o, ws_ml, ns, status_dev, s); break;
        }
    } else {
        switch (D) {
            case 64: e = gqa::launch_g<64, 64>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws_o, ws_ml, ns, status_dev, s); break;
            case 96: e = gqa::launch_g<96, 64>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws_o, ws_ml, ns, status_dev, s); break;
            default: e = gqa::launch_g<128, 64>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws_o, ws_ml, ns, status_dev, s); break;
        }
    }
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}
