// decode.cu -- single-token attention against the KV cache (split-K, HBM-bound).
//
// One query token per sequence attends over lens[b] cached keys: the KV-cache
// step of page "750美元从零训练3个LLM：一位开发者的实战复盘", section
// "V3：扩容与推理优化" (per-step cost O(n) instead of O(n^2)), batched as on page
// "从零手训LLaMa：125M模型11小时训练全记录"; the cache is read once per GQA group,
// never once per query head (first page, section "V2：引入前沿技术").
//
// Work: CTA (chunk, kv-head x head subgroup, b) covers 64 consecutive cache
// slots of one KV head and G of its query heads (CTAs past a sequence's length
// exit at once).  One thread issues three bulk copies -- the K chunk and the G
// query vectors on one barrier, the V chunk on another (each chunk is one
// contiguous block of the per-head slab) -- and about 33 KB of shared memory
// lets six CTAs share an SM, so the loads of some overlap the arithmetic of
// others.  Each of the four warps takes 16 of the chunk's keys through the
// whole step on its own:
//   1. score: 8 lanes per key, lane j holding 16-byte chunks j and j+8 of the row
//      against the G query vectors in registers (packed fma.f32x2); the 8 lanes
//      of a key read one contiguous 128-byte span (no bank conflicts) and three
//      xor-shuffles finish each dot product.  The V chunk keeps streaming in.
//   2. the warp's softmax statistics in base 2 by xor-shuffles: m_w, p, l_w.
//   3. p.V: each key's p is broadcast by a shuffle, lanes span D.
//   4. the four warp partials are merged (rescaled to their common maximum) and
//      the chunk's (m, l, o) go to the workspace.
// A second kernel, launched as a programmatic dependent of the first, merges
// the chunks of each (b, query head): M = max m_i,
// o = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i.  One warp per row, lanes
// spanning D; every partial of the row is loaded before any is used, and the
// kernel's few registers per CTA let all rows of a batch be resident at once,
// so the merge costs about one memory round trip.  (Merging inside the first
// kernel -- the last chunk to finish, found with an atomic ticket, merging the
// rest -- measured slower: every CTA then has to fence its partial writes;
// so did one thread-block cluster per row merging through distributed shared
// memory, and CTAs streaming several chunks through per-warp rings: fewer,
// longer-lived CTAs hide the copies' latency worse than many one-shot ones.)
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecCH = 64;            // cache slots per CTA
constexpr int kMaxG = 4;              // query heads per CTA, at most

template <int D, int G>
struct DecShape {
    static constexpr int CH = kDecCH;
    static constexpr int kKeysPerWarp = CH / kDecWarps;       // 16: four passes of 4 keys
    static constexpr int kPasses = kKeysPerWarp / 4;
    static constexpr int kRowChunks = D / 8;                  // 16-byte chunks per cache row
    static constexpr int kLaneChunks = (kRowChunks + 7) / 8;  // chunks per lane (8 lanes per key)
    static constexpr int kEPL = D == 64 ? 2 : 4;              // p.V elements per lane
    static constexpr int kPVLanes = D / kEPL;                 // 32, 24 or 32 active lanes
    static constexpr int kKVBytes = CH * D * 2;
    static constexpr int kQBytes = (G * D * 2 + 127) / 128 * 128;
    // [K | V | q][(m, l): warps x G x 2 f32]; the warps' partial outputs
    // (warps x G x D f32) are written over the K chunk once every warp has
    // finished its scores.
    static constexpr int kOffV = kKVBytes;
    static constexpr int kOffQ = 2 * kKVBytes;
    static constexpr int kOffML = kOffQ + kQBytes;
    static constexpr int kOffPartial = 0;
    static constexpr int kSmem = kOffML + kDecWarps * G * 2 * 4;
    static_assert(kDecWarps * G * D * 4 <= kKVBytes, "partials must fit over the K chunk");
};

// Workspace: [(m, l): rows x 2 f32][o: rows x D f32] with rows = B x Hq x n_splits,
// row (b, h, c) = (b * Hq + h) * n_splits + c.

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ kc,
              const uint16_t *__restrict__ vc, const int32_t *__restrict__ lens, int max_len,
              int Hq, int Hkv, int Lmax, float scale_log2, int n_splits, int n_sub,
              float *__restrict__ ws_ml, float *__restrict__ ws_o, int32_t *status) {
    using S = DecShape<D, G>;
    constexpr int CH = S::CH;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[2];     // [0]: K chunk + q, [1]: V chunk
    __shared__ float sw[kDecWarps * kMaxG];       // warp merge weights [warp][head]

    // Launched as a programmatic dependent of whatever precedes it on the stream
    // (normally the append that wrote lens and the new K/V slot): wait for it to
    // complete before reading anything it produced.  The merge kernel may then
    // be scheduled; it waits for this grid before it reads the partials.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int c = blockIdx.x;                     // chunk of the sequence
    const int kvh = blockIdx.y / n_sub, sub = blockIdx.y - kvh * n_sub;
    const int b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = Hq / Hkv;
    const int h0 = kvh * g + sub * G;             // first query head of this CTA
    const int len = lens[b];
    if (len < 1 || len > max_len || len > Lmax) {
        if (c == 0 && blockIdx.y == 0 && tid == 0)
            report(status, len < 1 ? GQA_DEV_BAD_LEN : GQA_DEV_CAPACITY);
        return;
    }
    const int key0 = c * CH;
    if (key0 >= len) return;
    const int nk = min(CH, len - key0);
    const uint32_t bar_k = ptx::smem_addr(&bars[0]);
    const uint32_t bar_v = ptx::smem_addr(&bars[1]);
    if (tid == 0) {
        ptx::mbar_init(bar_k, 1);
        ptx::mbar_init(bar_v, 1);
        ptx::fence_barrier_init();
        const uint32_t bytes = (uint32_t)nk * D * 2;
        const size_t slab = (((size_t)b * Hkv + kvh) * Lmax + key0) * D;
        const uint64_t pol = ptx::policy_evict_first();
        ptx::mbar_arrive_expect_tx(bar_k, bytes + G * D * 2);
        ptx::bulk_g2s_hint(ptx::smem_addr(smem), kc + slab, bytes, bar_k, pol);
        ptx::bulk_g2s(ptx::smem_addr(smem + S::kOffQ), q + ((size_t)b * Hq + h0) * D, G * D * 2,
                      bar_k);
        ptx::mbar_arrive_expect_tx(bar_v, bytes);
        ptx::bulk_g2s_hint(ptx::smem_addr(smem + S::kOffV), vc + slab, bytes, bar_v, pol);
    }
    __syncthreads();   // barriers initialised before anyone waits on them
    const uint16_t *ks = reinterpret_cast<const uint16_t *>(smem);
    const uint16_t *vs = reinterpret_cast<const uint16_t *>(smem + S::kOffV);
    const uint16_t *qs = reinterpret_cast<const uint16_t *>(smem + S::kOffQ);
    float *wml = reinterpret_cast<float *>(smem + S::kOffML);           // [warp][G][2]
    float *partial = reinterpret_cast<float *>(smem + S::kOffPartial);  // [warp][G][D]
    if (!__syncthreads_and(ptx::mbar_wait(bar_k, 0))) {
        // A copy that missed its deadline may still land in this CTA's shared
        // memory: give both one more bounded wait before the CTA retires.
        ptx::mbar_wait(bar_k, 0);
        ptx::mbar_wait(bar_v, 0);
        if (tid == 0) report(status, GQA_DEV_TIMEOUT);
        return;
    }

    const int j = lane & 7;          // lane within its key's group of 8
    const int kq = lane >> 3;        // key slot within a pass
    const int kw0 = warp * S::kKeysPerWarp;                  // this warp's first key
    const int kwn = max(0, min(S::kKeysPerWarp, nk - kw0));  // its live keys

    // ---- 1. scores: 8 lanes per key; lane j holds 16-byte chunks j, j+8 ----
    float qr[G][S::kLaneChunks][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < S::kLaneChunks; ++i) {
            const int cc = j + 8 * i;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (cc < S::kRowChunks) w = *reinterpret_cast<const uint4 *>(qs + h * D + cc * 8);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                qr[h][i][2 * e] = bf16lo(ww[e]);
                qr[h][i][2 * e + 1] = bf16hi(ww[e]);
            }
        }
    float sc[S::kPasses][G];
#pragma unroll
    for (int pass = 0; pass < S::kPasses; ++pass) {
        const int kl = pass * 4 + kq;                     // key within the warp's 16
        const uint16_t *krow = ks + (kw0 + kl) * D;
        float acc0[G], acc1[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc0[h] = acc1[h] = 0.f;
#pragma unroll
        for (int i = 0; i < S::kLaneChunks; ++i) {
            const int cc = j + 8 * i;
            if (cc < S::kRowChunks) {
                const uint4 w = *reinterpret_cast<const uint4 *>(krow + cc * 8);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float k0 = bf16lo(ww[e]), k1 = bf16hi(ww[e]);
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        ptx::ffma2(acc0[h], acc1[h], qr[h][i][2 * e], qr[h][i][2 * e + 1], k0, k1,
                                   acc0[h], acc1[h]);
                }
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float a = acc0[h] + acc1[h];
            a += __shfl_xor_sync(0xffffffffu, a, 1);
            a += __shfl_xor_sync(0xffffffffu, a, 2);
            a += __shfl_xor_sync(0xffffffffu, a, 4);
            sc[pass][h] = kl < kwn ? a * scale_log2 : -INFINITY;
        }
    }

    // ---- 2. the warp's own softmax statistics (base 2) ----
    float mw[G], lw[G], pw[S::kPasses][G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float m = sc[0][h];
#pragma unroll
        for (int pass = 1; pass < S::kPasses; ++pass) m = fmaxf(m, sc[pass][h]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        const float mref = m == -INFINITY ? 0.f : m;      // a warp with no live key
        float l = 0.f;
#pragma unroll
        for (int pass = 0; pass < S::kPasses; ++pass) {
            pw[pass][h] = ex2(sc[pass][h] - mref);
            l += pw[pass][h];                             // 8 lanes = one key
        }
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        mw[h] = m;
        lw[h] = l;
    }

    // ---- 3. p . V over the warp's live keys: lanes span D ----
    if (!__syncthreads_and(ptx::mbar_wait(bar_v, 0))) {
        ptx::mbar_wait(bar_v, 0);
        if (tid == 0) report(status, GQA_DEV_TIMEOUT);
        return;
    }
    float o[G][S::kEPL];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < S::kEPL; ++e) o[h][e] = 0.f;
#pragma unroll
    for (int kl = 0; kl < S::kKeysPerWarp; ++kl) {
        if (kl >= kwn) break;                             // warp-uniform
        float pk[G];
#pragma unroll
        for (int h = 0; h < G; ++h) pk[h] = __shfl_sync(0xffffffffu, pw[kl >> 2][h], (kl & 3) * 8);
        if (lane < S::kPVLanes) {
            const uint16_t *vrow = vs + (kw0 + kl) * D;
            float v[S::kEPL];
            if constexpr (S::kEPL == 4) {
                const uint2 w = *reinterpret_cast<const uint2 *>(vrow + lane * 4);
                v[0] = bf16lo(w.x);
                v[1] = bf16hi(w.x);
                v[2] = bf16lo(w.y);
                v[3] = bf16hi(w.y);
            } else {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(vrow + lane * 2);
                v[0] = bf16lo(w);
                v[1] = bf16hi(w);
            }
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < S::kEPL; e += 2)
                    ptx::ffma2(o[h][e], o[h][e + 1], pk[h], pk[h], v[e], v[e + 1], o[h][e],
                               o[h][e + 1]);
        }
    }
    if (lane < S::kPVLanes) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float *dst = partial + (warp * G + h) * D + lane * S::kEPL;
            if constexpr (S::kEPL == 4)
                *reinterpret_cast<float4 *>(dst) = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
            else
                *reinterpret_cast<float2 *>(dst) = make_float2(o[h][0], o[h][1]);
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            wml[(warp * G + h) * 2] = mw[h];
            wml[(warp * G + h) * 2 + 1] = lw[h];
        }
    }
    __syncthreads();

    // ---- 4. merge the warps; the chunk's (m, l, o) to the workspace ----
    const size_t row0 = ((size_t)b * Hq + h0) * n_splits + c;
    if (tid < G) {
        const int h = tid;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wml[(w * G + h) * 2]);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float mwv = wml[(w * G + h) * 2];
            const float f = mwv == -INFINITY ? 0.f : ex2(mwv - M);
            sw[w * kMaxG + h] = f;
            L = fmaf(f, wml[(w * G + h) * 2 + 1], L);
        }
        ws_ml[(row0 + (size_t)h * n_splits) * 2 + 0] = M;
        ws_ml[(row0 + (size_t)h * n_splits) * 2 + 1] = L;
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kDecThreads) {
        const int h = idx / D, d = idx - h * D;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w)
            acc = fmaf(sw[w * kMaxG + h], partial[(w * G + h) * D + d], acc);
        ws_o[(row0 + (size_t)h * n_splits) * D + d] = acc;
    }

}

// Merge the chunks of each (b, query head) row: one warp per row, four rows per
// CTA, lane i owning coordinates 4i .. 4i+3.  For up to 32 chunks at a time the
// lanes load every chunk's partial of their coordinates and lane i the chunk's
// (m, l), all before any is used; the maximum and the weights 2^(m_i - M) then
// travel by shuffle.  Rows of more than 32 chunks repeat this per group of 32,
// rescaling what the earlier groups summed (online, like the split kernel).
template <int D>
__global__ void __launch_bounds__(128)
decode_merge_kernel(const float *__restrict__ ws_ml, const float *__restrict__ ws_o,
                    const int32_t *__restrict__ lens, int max_len, int Hq, int Lmax,
                    int n_splits, int n_rows, uint16_t *__restrict__ out) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);   // b * Hq + h
    if (row >= n_rows) return;
    const int b = row / Hq;
    const int len = lens[b];
    uint16_t *o = out + (size_t)row * D;
    constexpr int kLanes = D / 4;
    const bool live = lane < kLanes;
    if (len < 1 || len > max_len || len > Lmax) {
        if (live) *reinterpret_cast<uint2 *>(o + lane * 4) = make_uint2(0, 0);
        return;
    }
    const int ns = (len + kDecCH - 1) / kDecCH;
    const float *ml = ws_ml + (size_t)row * n_splits * 2;
    const float *po = ws_o + (size_t)row * n_splits * D + lane * 4;
    float M = -INFINITY, L = 0.f;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int base = 0; base < ns; base += 32) {
        const int n = min(32, ns - base);
        float4 pv[32];
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
            pv[jj] = (live && jj < n)
                         ? *reinterpret_cast<const float4 *>(po + (size_t)(base + jj) * D)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        const float2 mi = lane < n ? *reinterpret_cast<const float2 *>(ml + 2 * (base + lane))
                                   : make_float2(-INFINITY, 0.f);
        const float mn = fmaxf(M, warp_max(mi.x));
        const float alpha = ex2(M - mn);          // 0 on the first group
        const float w = lane < n ? ex2(mi.x - mn) : 0.f;
        L = fmaf(L, alpha, warp_sum(w * mi.y));
        a0 *= alpha;
        a1 *= alpha;
        a2 *= alpha;
        a3 *= alpha;
        M = mn;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
            const float wj = __shfl_sync(0xffffffffu, w, jj);
            a0 = fmaf(wj, pv[jj].x, a0);
            a1 = fmaf(wj, pv[jj].y, a1);
            a2 = fmaf(wj, pv[jj].z, a2);
            a3 = fmaf(wj, pv[jj].w, a3);
        }
    }
    if (live) {
        const float inv = 1.f / L;
        *reinterpret_cast<uint2 *>(o + lane * 4) =
            make_uint2(pack_bf16x2(a0 * inv, a1 * inv), pack_bf16x2(a2 * inv, a3 * inv));
    }
}

template <int D, int G>
cudaError_t launch_decode(const void *q, const void *kc, const void *vc, const int32_t *lens,
                          int max_len, void *out, int B, int Hq, int Hkv, int Lmax,
                          float scale_log2, void *ws, int n_splits, int32_t *status,
                          cudaStream_t s) {
    using S = DecShape<D, G>;
    auto kern = decode_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::kSmem);
    if (e != cudaSuccess) return e;
    const int n_sub = (Hq / Hkv) / G;
    const size_t rows = (size_t)B * Hq * n_splits;
    float *ws_ml = static_cast<float *>(ws);
    float *ws_o = ws_ml + rows * 2;
    // Both launches are programmatic dependents of the kernel before them.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_splits, Hkv * n_sub, B);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = S::kSmem;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, static_cast<const uint16_t *>(q),
                           static_cast<const uint16_t *>(kc), static_cast<const uint16_t *>(vc),
                           lens, max_len, Hq, Hkv, Lmax, scale_log2, n_splits, n_sub, ws_ml, ws_o,
                           status);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)((B * Hq + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D>, (const float *)ws_ml, (const float *)ws_o,
                              lens, max_len, Hq, Lmax, n_splits, B * Hq, static_cast<uint16_t *>(out));
}

// Query heads per CTA: the largest of {3, 2, 1} (D = 128) or {4, 3, 2, 1}
// dividing the group size g, bounded by the registers the query vectors take.
int heads_per_cta(int g, int D) {
    const int cap = D == 128 ? 3 : 4;
    for (int G = cap; G > 1; --G)
        if (g % G == 0) return G;
    return 1;
}

template <int D>
cudaError_t launch_g(int G, const void *q, const void *kc, const void *vc, const int32_t *lens,
                     int max_len, void *out, int B, int Hq, int Hkv, int Lmax, float sl2,
                     void *ws, int ns, int32_t *st, cudaStream_t s) {
    switch (G) {
        case 1: return launch_decode<D, 1>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, ws, ns, st, s);
        case 2: return launch_decode<D, 2>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, ws, ns, st, s);
        case 3: return launch_decode<D, 3>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, ws, ns, st, s);
        default:
            if constexpr (D != 128)
                return launch_decode<D, 4>(q, kc, vc, lens, max_len, out, B, Hq, Hkv, Lmax, sl2, ws, ns, st, s);
            return cudaErrorInvalidValue;
    }
}

}  // namespace
}  // namespace gqa

extern "C" size_t gqa_decode_workspace_bytes(int B, int Hq, int D, int max_len) {
    if (B < 1 || Hq < 1 || max_len < 1 || !gqa_host::head_dim_ok(D)) return 0;
    const size_t ns = (size_t)(max_len + gqa::kDecCH - 1) / gqa::kDecCH;
    const size_t rows = (size_t)B * Hq * ns;
    return rows * 2 * 4 + rows * (size_t)D * 4;
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
    const int ns = (max_len_host + gqa::kDecCH - 1) / gqa::kDecCH;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
    const float sl2 = sc * 1.4426950408889634f;   // scores in base-2 units
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch (D) {
        case 64: e = gqa::launch_g<64>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws, ns, status_dev, s); break;
        case 96: e = gqa::launch_g<96>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws, ns, status_dev, s); break;
        default: e = gqa::launch_g<128>(G, q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, Lmax, sl2, ws, ns, status_dev, s); break;
    }
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// gqa_decode_noalloc: the same decode with its scratch in a fixed device array
// ---------------------------------------------------------------------------
// Some callers cannot hand this library any device scratch: a host framework
// that owns every byte of device memory and gives its plugins no allocator, or
// a serving loop that must not call cudaMalloc once it is running (the call
// synchronises the device and can fail when memory is tight).  For them the
// decode can keep its partial results in this file-scope array instead of a
// caller workspace.  The array is created with the module on every GPU that
// loads the library and lives until the process exits; the decode needs no
// part of it to start at zero.  Host code cannot use `g_noalloc_scratch` as an
// address (it names a host-side stand-in), so the array's device address is
// looked up with cudaGetSymbolAddress the first time a CUDA context calls, and
// kept for that context: the address belongs to the context the module was
// loaded into, so a caller that runs its own (non-primary) context on a device
// gets that context's copy, never another context's.
namespace {

constexpr size_t kNoAllocScratchBytes = GQA_DECODE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

constexpr int kMaxContexts = 64;
std::mutex g_noalloc_mutex;
CUcontext g_noalloc_ctx[kMaxContexts] = {};
void *g_noalloc_ptr[kMaxContexts] = {};
int g_noalloc_n = 0;

// Device address of the scratch array in the calling thread's current context.
gqa_status noalloc_scratch(void **ptr) {
    CtxGetCurrentFn cur = ctx_get_current();
    if (!cur) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    CUcontext ctx = nullptr;
    if (cur(&ctx) != CUDA_SUCCESS) return GQA_ERR_CUDA;
    for (int i = 0; ctx && i < g_noalloc_n; ++i)
        if (g_noalloc_ctx[i] == ctx) {
            *ptr = g_noalloc_ptr[i];
            return GQA_OK;
        }
    // First call from this context (with no context current yet, the runtime
    // makes the device's primary context current here).
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GQA_ERR_CUDA;
    if (cur(&ctx) != CUDA_SUCCESS || !ctx) return GQA_ERR_CUDA;
    if (g_noalloc_n < kMaxContexts) {
        g_noalloc_ctx[g_noalloc_n] = ctx;
        g_noalloc_ptr[g_noalloc_n] = p;
        ++g_noalloc_n;
    }
    *ptr = p;
    return GQA_OK;
}

}  // namespace

extern "C" gqa_status gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                         const int32_t *lens, int max_len_host, void *out, int B,
                                         int Hq, int Hkv, int D, int Lmax, float scale,
                                         int32_t *status_dev, void *stream) {
    if (B < 1 || Hq < 1 || max_len_host < 1 || !gqa_host::head_dim_ok(D))
        return gqa_host::head_dim_ok(D) ? GQA_ERR_INVALID_ARG : GQA_ERR_UNSUPPORTED;
    const size_t need = gqa_decode_workspace_bytes(B, Hq, D, max_len_host);
    if (need == 0 || need > kNoAllocScratchBytes) return GQA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const gqa_status st = noalloc_scratch(&scratch);
    if (st != GQA_OK) return st;
    return gqa_decode(q, k_cache, v_cache, lens, max_len_host, out, B, Hq, Hkv, D, Lmax, scale,
                      scratch, kNoAllocScratchBytes, status_dev, stream);
}
