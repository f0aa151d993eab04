// backward.cu -- the backward of causal GQA attention on the tcgen05 tensor cores.
//
// The pages' models train through the causal scaled_dot_product_attention
// (page "训练3.8B LLM至0.384 CORE，成本998美元 – Hugo Vergnes", sections "无效的方法"
// and "提高吞吐量"; page "Build a Large Language Model from Scratch", section 3.1),
// with query heads sharing K/V heads in groups (page "750美元从零训练3个LLM：一位
// 开发者的实战复盘", section "V2：引入前沿技术").  For one query head, with
// P = softmax(Q K^T * c) (causal, c the softmax scale) and the incoming gradient
// dO of the output O = P V:
//     dV = P^T dO,   dP = dO V^T,   dS = P * (dP - Delta),  Delta = rowsum(dO * O),
//     dQ = c dS K,   dK = c dS^T Q,
// and the K/V gradients of a KV head sum over the query heads of its group.  P is
// recomputed from the forward's row log-sum-exp, never stored.
//
// Three launches:
//   delta_kernel   Delta[b, h, t] = sum_d dO * O (HBM-bound, 16-byte loads, two
//                  rows per lane), and
//                  the exponent offset -lse[b, h, t] log2(e) the dK/dV kernel reads;
//   bwd_kv_kernel  per (b, KV head, 128-key tile j), persistent: for every query
//                  head of the group and every query tile i >= j, in halves of 64
//                  queries,
//                    S^T = K_j Q^T, dP^T = V_j dO^T            (two SS MMAs)
//                    P^T, dS^T in bf16 over S^T, dP^T in TMEM  (thread = key)
//                    dV_j += P^T dO, dK_j += dS^T Q             (two TS MMAs)
//                  dK_j and dV_j stay in tensor memory until the tile is done, so
//                  the group's sum needs no atomics;
//   bwd_q_kernel   per (b, query head, 128-query tile i), persistent: for every
//                  key tile j <= i,  S = Q_i K_j^T, dP = dO_i V_j^T, dS in bf16 over
//                  S, dQ_i += dS K_j.
// The dQ kernel needs only Delta, not dK / dV: the dK/dV kernel lets it launch
// right away (its CTAs take the SMs the dK/dV kernel's CTAs free), and it waits
// for the dK/dV kernel only before it exits, so the launch ends with both done.
// The dK/dV kernel keeps two halves in flight (S^T / dP^T double-buffered in
// tensor memory), so the tensor core works on one while the elementwise warps
// work on the other.  The dQ kernel keeps S in two buffers and a single dP that
// the warps release as soon as it is in registers, so S and dP of the next key
// tile run while the warps work on this one (K and V in separate rings, 3 and 2
// tiles deep, since K is held a step longer for dQ += dS K); the warps drain an
// item's dQ after the first key tile of their next item, so the wait for its
// last MMA overlaps that work, and they transpose 16-byte pieces within groups
// of four lanes so each store writes 64 contiguous bytes of eight rows.
// The same shared-memory tile serves as a K-major operand (the contraction over
// D) and as an MN-major one (the contraction over its rows), as in the forward
// kernel.  Warp roles (384 threads, three warpgroups): warps 0-7 elementwise +
// epilogue (thread = TMEM lane; warps w and w + 4 share lane quadrant w and take
// 64 of the 128 columns each; 208 registers), warp 8 TMA producer, warp 9 MMA
// issuer, warps 10-11 idle (88 registers), the forward kernel's roles.  Every mbarrier wait is
// bounded (1 s) and raises GQA_DEV_TIMEOUT; tensor memory is released only after
// the MMA thread has seen its last MMA complete.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace gqa {
namespace {

constexpr int kBwThreads = 384;
constexpr int kBwTmaWarp = 8;
constexpr int kBwMmaWarp = 9;
constexpr uint32_t kBwEwRegs = 208, kBwCtlRegs = 88;   // 2 * 208 + 88 = 3 * 168 at launch
static_assert(2 * kBwEwRegs + kBwCtlRegs == 3 * 168 && kBwThreads == 3 * 128,
              "register split must balance");
constexpr int kEwWarps = 8;                 // elementwise warps: 2 per TMEM lane quadrant
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwShape {
    static constexpr int kBlocks = (D + 63) / 64;           // 128-byte column blocks
    static constexpr int kBlockBytes = 128 * 128;           // 128 rows x 128 bytes
    static constexpr int kTileBytes = kBlocks * kBlockBytes;
    static constexpr int kKSteps = D / 16;
    static constexpr int kVecBytes = 128 * 4;               // 128 fp32 (lse or delta)
    static constexpr int kStages = 2;
    // dK/dV kernel: [K_j | V_j | stages of (Q_i | dO_i | lse_i | delta_i)]
    static constexpr int kStageBytes = 2 * kTileBytes + 2 * kVecBytes;   // multiple of 1024
    static constexpr int kOffStage = 2 * kTileBytes;
    static constexpr int kOffOut = kOffStage + kStages * kStageBytes;   // dK/dV staging, 64 columns
    static constexpr int kSmemKV = kOffOut + kBlockBytes + 1024;
    static_assert(kSmemKV <= 227 * 1024, "shared memory per CTA");
    // dK/dV kernel tensor memory: the score buffers, then the fp32 accumulators
    static constexpr uint32_t kColAcc0 = 256, kColAcc1 = 384;
};

struct BwMaps {
    CUtensorMap q, dout, k, v, lse, delta, dk, dv;
};

struct BwSync {                                 // the dK/dV kernel's barriers
    uint64_t fixed_full, fixed_empty;          // K_j, V_j
    uint64_t st_full[2], st_empty[2];          // the ring of (Q_i, dO_i, lse_i, Delta_i)
    uint64_t acc_full, acc_empty;              // dK, dV accumulated / read out
    uint64_t h_full[2], h_done[2];             // two 64-query halves
    uint64_t mma_done;
    uint32_t tmem_base;
};

struct BwGrid {
    int B, T, Hq, Hkv, nT, n_items, lse_stride;
    float scale_log2, scale;
    const float *lse, *delta;
    uint16_t *d0, *d1;                          // dK, dV (dK/dV kernel) or dQ (dQ kernel)
    int Lmax;
};

__device__ __forceinline__ uint32_t A(const uint64_t &b) { return ptx::smem_addr(&b); }

// d = a * b on a pair of floats (one f32x2 instruction).
__device__ __forceinline__ void fmul2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Bring a tile of a 4-D tensor into L2 ahead of its load (no shared memory, no barrier).
__device__ __forceinline__ void l2_prefetch_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];"
                 ::"l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3) : "memory");
}

// The k-th item of this CTA: items are numbered longest first and dealt out in
// rounds of gridDim.x in snake order (every other round backwards).
__device__ __forceinline__ int bw_w(int k) {
    const int G = gridDim.x, c = blockIdx.x;
    return k * G + ((k & 1) ? G - 1 - c : c);
}

template <int D>
struct BwMma {
    using S = BwShape<D>;
    // D(tmem) = A(smem, K-major 128 x D) . B(smem, K-major 128 x D)^T : 128 x 128
    static __device__ __forceinline__ void ss(uint32_t go, uint32_t d, uint32_t a, uint32_t b) {
        constexpr uint32_t id = ptx::idesc_bf16_f32(128, 128, false);
#pragma unroll
        for (int ks = 0; ks < S::kKSteps; ++ks) {
            const uint32_t off = (ks >> 2) * S::kBlockBytes + (ks & 3) * 32;
            ptx::mma_ss_if(go, d, ptx::smem_desc_sw128(a + off, 16, 1024),
                        ptx::smem_desc_sw128(b + off, 16, 1024), id, ks > 0);
        }
    }
    // D(tmem, 128 x D) (+)= A(tmem, bf16 128 x 128) . B(smem, 128 rows x D, MN-major)
    static __device__ __forceinline__ void ts(uint32_t go, uint32_t d, uint32_t a_tmem, uint32_t b, bool acc) {
        constexpr uint32_t id = ptx::idesc_bf16_f32(128, D, true);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            ptx::mma_ts_if(go, d, a_tmem + ks * 8, ptx::smem_desc_sw128(b + ks * 2048, S::kBlockBytes, 1024),
                        id, (acc || ks > 0) ? 1u : 0u);
    }
};

// MMAs on halves of a 128-row tile (64 rows at a time), for the dK/dV pipeline.
template <int D>
struct BwMmaHalf {
    using S = BwShape<D>;
    // D(tmem, 128 x 64) = A(smem, K-major 128 x D) . B(smem, 64 rows of a K-major tile)^T
    static __device__ __forceinline__ void ss(uint32_t go, uint32_t d, uint32_t a, uint32_t b) {
        constexpr uint32_t id = ptx::idesc_bf16_f32(128, 64, false);
#pragma unroll
        for (int ks = 0; ks < S::kKSteps; ++ks) {
            const uint32_t off = (ks >> 2) * S::kBlockBytes + (ks & 3) * 32;
            ptx::mma_ss_if(go, d, ptx::smem_desc_sw128(a + off, 16, 1024),
                        ptx::smem_desc_sw128(b + off, 16, 1024), id, ks > 0);
        }
    }
    // D(tmem, 128 x D) (+)= A(tmem, bf16 128 x 64) . B(smem, 64 rows x D, MN-major)
    static __device__ __forceinline__ void ts(uint32_t go, uint32_t d, uint32_t a_tmem, uint32_t b, bool acc) {
        constexpr uint32_t id = ptx::idesc_bf16_f32(128, D, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            ptx::mma_ts_if(go, d, a_tmem + ks * 8, ptx::smem_desc_sw128(b + ks * 2048, S::kBlockBytes, 1024),
                        id, (acc || ks > 0) ? 1u : 0u);
    }
};

// ---------------------------------------------------------------------------
// Delta = rowsum(dO * O): TPR lanes per (t, h) row of sequence blockIdx.y, 16-byte
// loads, kPasses rows per lane with all their loads issued before the first sum
// ---------------------------------------------------------------------------
template <int D, int kPasses>
__global__ void __launch_bounds__(256)
delta_kernel(const uint16_t *__restrict__ out, const uint16_t *__restrict__ dout,
             const float *__restrict__ lse, float *__restrict__ delta, float *__restrict__ nl2,
             int T, int Hq, int stride) {
    constexpr int kChunks = D / 8;                       // 16-byte pieces per row
    constexpr int kTPR = kChunks > 8 ? 16 : 8;            // lanes per row (power of two)
    constexpr int kRowsPerPass = 256 / kTPR;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int j = threadIdx.x % kTPR, b = blockIdx.y;
    const int n_rows = T * Hq;                           // rows (t, h) of sequence b
    const int r0 = blockIdx.x * (kRowsPerPass * kPasses) + threadIdx.x / kTPR;
    const uint16_t *ob = out + (size_t)b * n_rows * D, *gb = dout + (size_t)b * n_rows * D;
    // every pass's loads are issued before the first is used
    uint4 a[kPasses], c[kPasses];
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const int r = r0 + p * kRowsPerPass;
        if (r < n_rows && j < kChunks) {
            a[p] = __ldcs(reinterpret_cast<const uint4 *>(ob + (size_t)r * D + 8 * j));
            c[p] = *reinterpret_cast<const uint4 *>(gb + (size_t)r * D + 8 * j);
        } else {
            a[p] = c[p] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const uint32_t aw[4] = {a[p].x, a[p].y, a[p].z, a[p].w}, cw[4] = {c[p].x, c[p].y, c[p].z, c[p].w};
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc = fmaf(bf16lo(aw[e]), bf16lo(cw[e]), acc);
            acc = fmaf(bf16hi(aw[e]), bf16hi(cw[e]), acc);
        }
#pragma unroll
        for (int o = kTPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        const int r = r0 + p * kRowsPerPass;
        if (r < n_rows && j == 0) {
            const int t = r / Hq, h = r - t * Hq;
            const size_t off = ((size_t)b * Hq + h) * stride + t;
            delta[off] = acc;
            nl2[off] = -lse[off] * kLog2e;          // the exponent's offset, base 2
        }
    }
}

// ---------------------------------------------------------------------------
// dK, dV: item = (b, KV head, key tile j), longest first (j ascending)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void kv_item(int w, const BwGrid &g, int &b, int &kvh, int &j) {
    const int per = g.B * g.Hkv;
    j = w / per;
    const int rest = w - j * per;
    b = rest / g.Hkv;
    kvh = rest - b * g.Hkv;
}

template <int D>
__device__ void kv_producer(const BwMaps &maps, BwSync &sy, uint8_t *smem, const BwGrid &g,
                            int32_t *status) {
    using S = BwShape<D>;
    const int grp = g.Hq / g.Hkv;
    int ic = 0, sc = 0;
    bool ok = true;
    for (int kk = 0, w = bw_w(0); w < g.n_items && ok; w = bw_w(++kk)) {
        int b, kvh, j;
        kv_item(w, g, b, kvh, j);
        ok = ptx::mbar_wait(A(sy.fixed_empty), (ic & 1) ^ 1);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(A(sy.fixed_full), 2 * S::kTileBytes);
        for (int kb = 0; kb < S::kBlocks; ++kb) {
            ptx::tma_load_3d(ptx::smem_addr(smem + kb * S::kBlockBytes), &maps.k, A(sy.fixed_full),
                             kb * 64, j * 128, b * g.Hkv + kvh);
            ptx::tma_load_3d(ptx::smem_addr(smem + S::kTileBytes + kb * S::kBlockBytes), &maps.v,
                             A(sy.fixed_full), kb * 64, j * 128, b * g.Hkv + kvh);
        }
        ++ic;
        for (int hh = 0; hh < grp && ok; ++hh) {
            const int h = kvh * grp + hh;
            for (int i = j; i < g.nT; ++i) {
                const int st = sc % S::kStages;
                ok = ptx::mbar_wait(A(sy.st_empty[st]), ((sc / S::kStages) & 1) ^ 1);
                if (!ok) break;
                uint8_t *base = smem + S::kOffStage + st * S::kStageBytes;
                const uint32_t bar = A(sy.st_full[st]);
                ptx::mbar_arrive_expect_tx(bar, 2 * S::kTileBytes + 2 * S::kVecBytes);
                for (int kb = 0; kb < S::kBlocks; ++kb) {
                    ptx::tma_load_4d(ptx::smem_addr(base + kb * S::kBlockBytes), &maps.q, bar,
                                     kb * 64, h, i * 128, b);
                    ptx::tma_load_4d(ptx::smem_addr(base + S::kTileBytes + kb * S::kBlockBytes),
                                     &maps.dout, bar, kb * 64, h, i * 128, b);
                }
                ptx::tma_load_2d(ptx::smem_addr(base + 2 * S::kTileBytes), &maps.lse, bar, i * 128,
                                 b * g.Hq + h);
                ptx::tma_load_2d(ptx::smem_addr(base + 2 * S::kTileBytes + S::kVecBytes), &maps.delta,
                                 bar, i * 128, b * g.Hq + h);
                ++sc;
            }
        }
    }
    if (!ok) {
        report(status, GQA_DEV_TIMEOUT);
        if (ic > 0) ptx::mbar_wait(A(sy.fixed_full), (ic - 1) & 1);
        for (int s = (sc > S::kStages ? sc - S::kStages : 0); s < sc; ++s)
            ptx::mbar_wait(A(sy.st_full[s % S::kStages]), (s / S::kStages) & 1);
    }
}

// The tile's queries are taken in two halves of 64 with S^T / dP^T of half u in
// tensor-memory buffer u % 2 (columns [128 (u % 2), 128 (u % 2) + 128): S^T then
// dP^T, 64 columns each), so the tensor core computes dV/dK of one half and
// S^T/dP^T of the next while the elementwise warps work on the other half.
template <int D>
__device__ void kv_mma(BwSync &sy, uint8_t *smem, uint32_t tmem, const BwGrid &g, int32_t *status) {
    using S = BwShape<D>;
    using M = BwMmaHalf<D>;
    const int grp = g.Hq / g.Hkv;
    const uint32_t k_base = ptx::smem_addr(smem), v_base = k_base + S::kTileBytes;
    int ic = 0, sc = 0, hc = 0, ac = 0;    // items, stages and halves consumed, accumulators
    bool ok = true;
    const uint32_t go = ptx::elect_one();   // the lane that issues
    auto stage_base = [&](int st) {
        return ptx::smem_addr(smem + S::kOffStage + st * S::kStageBytes);
    };
    // S^T / dP^T of half u (stage st, 64-row half h) into buffer u % 2
    auto issue_scores = [&](int u, int st, int h) {
        const uint32_t buf = tmem + 128 * (u & 1);
        const uint32_t qb = stage_base(st) + h * 64 * 128;
        M::ss(go, buf, k_base, qb);                          // S^T  = K_j Q_half^T
        M::ss(go, buf + 64, v_base, qb + S::kTileBytes);     // dP^T = V_j dO_half^T
        ptx::mma_commit_if(go, A(sy.h_full[u & 1]));
    };
    for (int kk = 0, w = bw_w(0); w < g.n_items && ok; w = bw_w(++kk)) {
        int b, kvh, j;
        kv_item(w, g, b, kvh, j);
        ok = ptx::mbar_wait_warp(A(sy.fixed_full), ic & 1);
        if (!ok) break;
        ++ic;
        ptx::tc_fence_after();
        const int n_half = 2 * grp * (g.nT - j);        // halves of this item
        const int sc0 = sc;
        // prologue: the scores of the first two halves (one stage)
        ok = ptx::mbar_wait_warp(A(sy.st_full[sc0 % S::kStages]), (sc0 / S::kStages) & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_scores(hc, sc0 % S::kStages, 0);
        issue_scores(hc + 1, sc0 % S::kStages, 1);
        for (int x = 0; x < n_half && ok; ++x) {
            const int u = hc + x;
            const int st = (sc0 + x / 2) % S::kStages;
            ok = ptx::mbar_wait_warp(A(sy.h_done[u & 1]), (u >> 1) & 1);   // P^T, dS^T of half u
            if (!ok) break;
            if (x == 0) {       // the previous item's epilogue has read dK, dV
                ok = ptx::mbar_wait_warp(A(sy.acc_empty), (ac & 1) ^ 1);
                if (!ok) break;
            }
            ptx::tc_fence_after();
            const uint32_t buf = tmem + 128 * (u & 1);
            const uint32_t qb = stage_base(st) + (x & 1) * 64 * 128;
            M::ts(go, tmem + S::kColAcc0, buf + 16, qb + S::kTileBytes, x > 0);   // dV += P^T dO_half
            M::ts(go, tmem + S::kColAcc1, buf + 80, qb, x > 0);                   // dK += dS^T Q_half
            if (x & 1) ptx::mma_commit_if(go, A(sy.st_empty[st]));              // both halves done
            // the scores of half u + 2 go into the buffer just consumed
            if (x + 2 < n_half) {
                const int st2 = (sc0 + (x + 2) / 2) % S::kStages;
                if (!(x & 1)) {
                    ok = ptx::mbar_wait_warp(A(sy.st_full[st2]), ((sc0 + (x + 2) / 2) / S::kStages) & 1);
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                issue_scores(u + 2, st2, x & 1);
            }
        }
        if (!ok) break;
        hc += n_half;
        sc += n_half / 2;
        ptx::mma_commit_if(go, A(sy.acc_full));
        ptx::mma_commit_if(go, A(sy.fixed_empty));
        ++ac;
    }
    if (!ok && go) report(status, GQA_DEV_TIMEOUT);
    ptx::mma_commit_if(go, A(sy.mma_done));
    ptx::mbar_wait_warp(A(sy.mma_done), 0);
}

// Elementwise work of the dK/dV kernel on one 64-query half: thread = key row r
// of tile j; warp w takes lane quadrant w % 4 and the half's columns
// [32 (w / 4), 32 (w / 4) + 32).  P^T and dS^T (packed bf16) go to columns
// [16, 48) and [80, 112) of the half's buffer: each warp writes only columns it
// has itself loaded (S^T [32 p, 32 p + 32) -> P^T [16 + 16 p, 32 + 16 p), and
// likewise for dP^T), so the two warps of a quadrant need no barrier.  Pairs of
// elements go through the f32x2 instructions.
template <int D, bool kEdge>
__device__ __forceinline__ void kv_block(const uint32_t (&sv)[32], const uint32_t (&dv)[32],
                                         const float *nl_v, const float *del_v, int qbase,
                                         int key, int T, float sl2, uint32_t (&pp)[16],
                                         uint32_t (&dd)[16]) {
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4) {
        const float4 l4 = *reinterpret_cast<const float4 *>(nl_v + 4 * c4);   // -lse log2(e)
        const float4 d4 = *reinterpret_cast<const float4 *>(del_v + 4 * c4);
        const float nl[4] = {l4.x, l4.y, l4.z, l4.w};
        const float dl[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = 4 * c4 + 2 * h;
            float x0, x1, y0, y1, d0, d1;
            ptx::ffma2(x0, x1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), sl2, sl2,
                       nl[2 * h], nl[2 * h + 1]);
            float p0 = ex2(x0), p1 = ex2(x1);
            if (kEdge) {
                const int query = qbase + e;
                if (query < key || query >= T) p0 = 0.f;
                if (query + 1 < key || query + 1 >= T) p1 = 0.f;
            }
            ptx::fsub2(y0, y1, __uint_as_float(dv[e]), __uint_as_float(dv[e + 1]), dl[2 * h],
                       dl[2 * h + 1]);
            fmul2(d0, d1, p0, p1, y0, y1);
            pp[e / 2] = pack_bf16x2(p0, p1);
            dd[e / 2] = pack_bf16x2(d0, d1);
        }
    }
}

template <int D>
__device__ void kv_elementwise(const BwMaps &maps, BwSync &sy, uint8_t *smem, uint32_t tmem,
                               const BwGrid &g, int32_t *status) {
    using S = BwShape<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int grp = g.Hq / g.Hkv;
    int hc = 0, sc = 0, ac = 0;
    bool ok = true;
    const bool st_issuer = threadIdx.x == 0;      // stores the staged dK / dV blocks
    for (int kk = 0, w = bw_w(0); w < g.n_items && ok; w = bw_w(++kk)) {
        int b, kvh, j;
        kv_item(w, g, b, kvh, j);
        const int key = j * 128 + r;
        const int n_half = 2 * grp * (g.nT - j);
        // half x is the (x & 1) half of query tile i, which runs j .. nT - 1 once
        // per query head of the group (counted, not divided: a division here
        // waits on the special-function unit behind the exponentials)
        for (int x = 0, i = j; x < n_half && ok; i = (x & 1) ? (i + 1 == g.nT ? j : i + 1) : i, ++x) {
            const int u = hc + x;
            const int st = (sc + x / 2) % S::kStages;
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.h_full[u & 1]), (u >> 1) & 1));
            if (!ok) break;
            ptx::tc_fence_after();
            const int col = 64 * (x & 1) + 32 * part;          // first query column of this warp
            const float *nl_v = reinterpret_cast<const float *>(      // -lse log2(e)
                smem + S::kOffStage + st * S::kStageBytes + 2 * S::kTileBytes) + col;
            const float *del_v = nl_v + 128;
            const uint32_t buf = lane_addr + 128 * (u & 1);
            uint32_t sv[32], dv[32];
            ptx::tmem_ld32(buf + 32 * part, sv);
            ptx::tmem_ld32(buf + 64 + 32 * part, dv);
            ptx::tmem_wait_ld();
            uint32_t pp[16], dd[16];
            if (i == j || (i + 1) * 128 > g.T)                   // some (query, key) masked
                kv_block<D, true>(sv, dv, nl_v, del_v, i * 128 + col, key, g.T, g.scale_log2, pp, dd);
            else
                kv_block<D, false>(sv, dv, nl_v, del_v, i * 128 + col, key, g.T, g.scale_log2, pp, dd);
            ptx::tmem_st16(buf + 16 + 16 * part, pp);
            ptx::tmem_st16(buf + 80 + 16 * part, dd);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(A(sy.h_done[u & 1]));
        }
        if (!ok) break;
        hc += n_half;
        sc += n_half / 2;
        // epilogue: dV_j and c dK_j rows to global memory, half of D per warp
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.acc_full), ac & 1));
        if (!ok) break;
        ++ac;
        ptx::tc_fence_after();
        const size_t row = ((size_t)b * g.Hkv + kvh) * g.Lmax + key;
        if ((j + 1) * 128 <= g.T) {
            // a whole key tile: dV, then c dK, 64 columns at a time through the
            // staging (128-byte swizzle; warp part p writes the block's columns
            // [32 p, 32 p + 32) of its row), stored by one thread with the tensor map
            uint8_t *stg = smem + S::kOffOut;
#pragma unroll
            for (int blk = 0; blk < 2 * S::kBlocks; ++blk) {
                const int tsr = blk / S::kBlocks, cb = blk % S::kBlocks;   // 0: dV, 1: dK
                const int c = 2 * cb + part;                               // 32-column chunk
                uint32_t w[16] = {};
                if (32 * c < D) {
                    uint32_t a[32];
                    ptx::tmem_ld32(lane_addr + (tsr ? S::kColAcc1 : S::kColAcc0) + 32 * c, a);
                    ptx::tmem_wait_ld();
                    const float f = tsr ? g.scale : 1.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(a[2 * e]) * f, __uint_as_float(a[2 * e + 1]) * f);
                }
                if (st_issuer) ptx::bulk_wait_read0();   // the last store has read the staging
                ptx::named_bar_sync(2, kEwWarps * 32);
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int ch = 4 * part + y;                              // 16-byte chunk of the row
                    *reinterpret_cast<uint4 *>(stg + r * 128 + ((ch ^ (r & 7)) << 4)) =
                        make_uint4(w[4 * y], w[4 * y + 1], w[4 * y + 2], w[4 * y + 3]);
                }
                ptx::fence_proxy_async_shared();
                ptx::named_bar_sync(2, kEwWarps * 32);
                if (st_issuer) {
                    ptx::tma_store_3d(tsr ? &maps.dk : &maps.dv, ptx::smem_addr(stg), 64 * cb, j * 128,
                                      b * g.Hkv + kvh);
                    ptx::bulk_commit();
                }
            }
        } else {
            // the ragged last key tile: its rows below T, straight from registers
            for (int c = part; c < D / 32; c += 2) {
                uint32_t va[32], ka[32];
                ptx::tmem_ld32(lane_addr + S::kColAcc0 + 32 * c, va);
                ptx::tmem_ld32(lane_addr + S::kColAcc1 + 32 * c, ka);
                ptx::tmem_wait_ld();
                uint32_t wv[16], wk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    wv[e] = pack_bf16x2(__uint_as_float(va[2 * e]), __uint_as_float(va[2 * e + 1]));
                    wk[e] = pack_bf16x2(__uint_as_float(ka[2 * e]) * g.scale,
                                        __uint_as_float(ka[2 * e + 1]) * g.scale);
                }
                if (key < g.T) {
                    uint4 *dvp = reinterpret_cast<uint4 *>(g.d1 + row * D + 32 * c);
                    uint4 *dkp = reinterpret_cast<uint4 *>(g.d0 + row * D + 32 * c);
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        dvp[y] = make_uint4(wv[4 * y], wv[4 * y + 1], wv[4 * y + 2], wv[4 * y + 3]);
                        dkp[y] = make_uint4(wk[4 * y], wk[4 * y + 1], wk[4 * y + 2], wk[4 * y + 3]);
                    }
                }
            }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(A(sy.acc_empty));
    }
    if (st_issuer) ptx::bulk_wait0();          // the dK / dV stores have completed
    if (!ok && lane == 0) report(status, GQA_DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
// dQ: item = (b, query head, query tile i), longest first (i descending)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void q_item(int w, const BwGrid &g, int &b, int &h, int &i) {
    const int per = g.B * g.Hq;
    const int ii = w / per;
    const int rest = w - ii * per;
    i = g.nT - 1 - ii;
    b = rest / g.Hq;
    h = rest - b * g.Hq;
}

// The dQ kernel's shared memory: [Q_i | dO_i | K ring (3 tiles) | V ring (2 tiles)],
// and its tensor memory: S in two buffers [0,128) and [128,256) (dS is written
// over the S it came from, packed bf16 in the buffer's columns [32, 96): each
// warp writes only columns it has loaded, so no barrier), dP [256, 384), the dQ
// accumulator [384, 384 + D).
template <int D>
struct BwQShape {
    using S = BwShape<D>;
    static constexpr int kStagesK = 3, kStagesV = 2;
    static constexpr int kOffK = 2 * S::kTileBytes;
    static constexpr int kOffV = kOffK + kStagesK * S::kTileBytes;
    static constexpr int kSmem = kOffV + kStagesV * S::kTileBytes + 1024;
    static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
    static constexpr uint32_t kColDP = 256, kColAcc = 384;
};

struct BwQSync {
    uint64_t fixed_full, fixed_empty;          // Q_i, dO_i
    uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
    uint64_t s_full[2], dp_full;               // S(u) in buffer u % 2; dP(u)
    uint64_t dp_free;                          // dP(u) read into registers
    uint64_t ds_full[2];                       // dS(u) written over S(u)
    uint64_t acc_full, acc_empty;
    uint64_t mma_done;
    uint32_t tmem_base;
};

template <int D>
__device__ void q_producer(const BwMaps &maps, BwQSync &sy, uint8_t *smem, const BwGrid &g,
                           int32_t *status) {
    using S = BwShape<D>;
    using Q = BwQShape<D>;
    const int grp = g.Hq / g.Hkv;
    int ic = 0, kc = 0, vc = 0;
    bool ok = true;
    for (int kk = 0, w = bw_w(0); w < g.n_items && ok; w = bw_w(++kk)) {
        int b, h, i;
        q_item(w, g, b, h, i);
        const int kvh = h / grp;
        ok = ptx::mbar_wait(A(sy.fixed_empty), (ic & 1) ^ 1);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(A(sy.fixed_full), 2 * S::kTileBytes);
        for (int kb = 0; kb < S::kBlocks; ++kb) {
            ptx::tma_load_4d(ptx::smem_addr(smem + kb * S::kBlockBytes), &maps.q, A(sy.fixed_full),
                             kb * 64, h, i * 128, b);
            ptx::tma_load_4d(ptx::smem_addr(smem + S::kTileBytes + kb * S::kBlockBytes), &maps.dout,
                             A(sy.fixed_full), kb * 64, h, i * 128, b);
        }
        ++ic;
        if (bw_w(kk + 1) < g.n_items) {     // the next item's Q / dO into L2
            int b2, h2, i2;
            q_item(bw_w(kk + 1), g, b2, h2, i2);
            for (int kb = 0; kb < S::kBlocks; ++kb) {
                l2_prefetch_4d(&maps.q, kb * 64, h2, i2 * 128, b2);
                l2_prefetch_4d(&maps.dout, kb * 64, h2, i2 * 128, b2);
            }
        }
        // K tiles run ahead of V tiles: S(u) needs K(u) before dP(u) needs V(u), and
        // K(u) is held until dQ(u), a step after V(u) is released.
        int jk = 0, jv = 0;
        while (ok && jv <= i) {
            if (jk <= i && jk < jv + Q::kStagesK) {
                const int st = kc % Q::kStagesK;
                ok = ptx::mbar_wait(A(sy.k_empty[st]), ((kc / Q::kStagesK) & 1) ^ 1);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(A(sy.k_full[st]), S::kTileBytes);
                for (int kb = 0; kb < S::kBlocks; ++kb)
                    ptx::tma_load_3d(ptx::smem_addr(smem + Q::kOffK + st * S::kTileBytes + kb * S::kBlockBytes),
                                     &maps.k, A(sy.k_full[st]), kb * 64, jk * 128, b * g.Hkv + kvh);
                ++kc;
                ++jk;
            }
            if (jv < jk) {
                const int st = vc % Q::kStagesV;
                ok = ptx::mbar_wait(A(sy.v_empty[st]), ((vc / Q::kStagesV) & 1) ^ 1);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(A(sy.v_full[st]), S::kTileBytes);
                for (int kb = 0; kb < S::kBlocks; ++kb)
                    ptx::tma_load_3d(ptx::smem_addr(smem + Q::kOffV + st * S::kTileBytes + kb * S::kBlockBytes),
                                     &maps.v, A(sy.v_full[st]), kb * 64, jv * 128, b * g.Hkv + kvh);
                ++vc;
                ++jv;
            }
        }
    }
    if (!ok) {
        report(status, GQA_DEV_TIMEOUT);
        if (ic > 0) ptx::mbar_wait(A(sy.fixed_full), (ic - 1) & 1);
        for (int j = (kc > Q::kStagesK ? kc - Q::kStagesK : 0); j < kc; ++j)
            ptx::mbar_wait(A(sy.k_full[j % Q::kStagesK]), (j / Q::kStagesK) & 1);
        for (int j = (vc > Q::kStagesV ? vc - Q::kStagesV : 0); j < vc; ++j)
            ptx::mbar_wait(A(sy.v_full[j % Q::kStagesV]), (j / Q::kStagesV) & 1);
    }
}

// The MMA thread walks the CTA's key tiles u (all items in turn).  Step u issues
// S(u) into buffer u % 2 (free: dQ(u - 2) read it earlier in the same queue),
// then dP(u) once the elementwise warps hold dP(u - 1) in registers, then
// dQ(u - 1) += dS(u - 1) K once they have written dS(u - 1).  So S(u) and dP(u)
// run while the warps work on tile u - 1.  At an item's first tile the
// previous item's last dQ goes first (its epilogue waits for it).
template <int D>
__device__ void q_mma(BwQSync &sy, uint8_t *smem, uint32_t tmem, const BwGrid &g, int32_t *status) {
    using S = BwShape<D>;
    using Q = BwQShape<D>;
    using M = BwMma<D>;
    const uint32_t q_base = ptx::smem_addr(smem), do_base = q_base + S::kTileBytes;
    const uint32_t k_base = ptx::smem_addr(smem + Q::kOffK), v_base = ptx::smem_addr(smem + Q::kOffV);
    int ic = 0, ac = 0;
    int u = 0;                    // key tiles of this CTA so far
    bool prev_first = false;      // tile u - 1 was the first of its item
    bool ok = true;
    const uint32_t go = ptx::elect_one();   // the lane that issues
    // dQ(u - 1): needs dS(u - 1); the item's first tile also needs the accumulator
    // drained by the previous item's epilogue; the item's last one completes dQ
    auto issue_dq = [&](int t, bool first, bool last) {
        if (!ptx::mbar_wait_warp(A(sy.ds_full[t & 1]), (t >> 1) & 1)) return false;
        if (first && !ptx::mbar_wait_warp(A(sy.acc_empty), (ac & 1) ^ 1)) return false;
        ptx::tc_fence_after();
        M::ts(go, tmem + Q::kColAcc, tmem + 128 * (t & 1) + 32, k_base + (t % Q::kStagesK) * S::kTileBytes,
              !first);
        ptx::mma_commit_if(go, A(sy.k_empty[t % Q::kStagesK]));
        if (last) {
            ptx::mma_commit_if(go, A(sy.acc_full));
            ++ac;
        }
        return true;
    };
    bool prev_last = false;
    for (int kk = 0, w = bw_w(0); w < g.n_items && ok; w = bw_w(++kk)) {
        int b, h, i;
        q_item(w, g, b, h, i);
        for (int j = 0; j <= i && ok; ++j, ++u) {
            if (j == 0) {
                if (u > 0) {
                    ok = issue_dq(u - 1, prev_first, prev_last);
                    if (!ok) break;
                }
                ok = ptx::mbar_wait_warp(A(sy.fixed_full), ic & 1);
                if (!ok) break;
                ++ic;
            }
            const int ks = u % Q::kStagesK, vs = u % Q::kStagesV;
            ok = ptx::mbar_wait_warp(A(sy.k_full[ks]), (u / Q::kStagesK) & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            M::ss(go, tmem + 128 * (u & 1), q_base, k_base + ks * S::kTileBytes);     // S = Q_i K_j^T
            ptx::mma_commit_if(go, A(sy.s_full[u & 1]));
            ok = ptx::mbar_wait_warp(A(sy.v_full[vs]), (u / Q::kStagesV) & 1);
            if (ok && u > 0 && j > 0) ok = ptx::mbar_wait_warp(A(sy.dp_free), (u - 1) & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            M::ss(go, tmem + Q::kColDP, do_base, v_base + vs * S::kTileBytes);      // dP = dO_i V_j^T
            ptx::mma_commit_if(go, A(sy.dp_full));
            ptx::mma_commit_if(go, A(sy.v_empty[vs]));
            if (j == i) ptx::mma_commit_if(go, A(sy.fixed_empty));                      // Q_i, dO_i read
            if (j > 0) {
                ok = issue_dq(u - 1, prev_first, prev_last);
                if (!ok) break;
            }
            prev_first = j == 0;
            prev_last = j == i;
        }
    }
    if (ok && u > 0) ok = issue_dq(u - 1, prev_first, prev_last);
    if (!ok && go) report(status, GQA_DEV_TIMEOUT);
    ptx::mma_commit_if(go, A(sy.mma_done));
    ptx::mbar_wait_warp(A(sy.mma_done), 0);
}

template <bool kDiag>
__device__ __forceinline__ void q_block(const uint32_t (&sv)[64], const uint32_t (&dv)[64],
                                        int key0, int qrow, float sl2, float lse2, float dlt,
                                        uint32_t (&dd)[32]) {
#pragma unroll
    for (int e2 = 0; e2 < 32; ++e2) {
        const int e = 2 * e2;
        float x0, x1, y0, y1, d0, d1;
        ptx::ffma2(x0, x1, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]), sl2, sl2, -lse2,
                   -lse2);
        float p0 = ex2(x0), p1 = ex2(x1);
        if (kDiag) {
            if (key0 + e > qrow) p0 = 0.f;
            if (key0 + e + 1 > qrow) p1 = 0.f;
        }
        ptx::fsub2(y0, y1, __uint_as_float(dv[e]), __uint_as_float(dv[e + 1]), dlt, dlt);
        fmul2(d0, d1, p0, p1, y0, y1);
        dd[e2] = pack_bf16x2(d0, d1);
    }
}

__device__ __forceinline__ uint4 shfl_xor_u4(uint4 v, int m) {
    v.x = __shfl_xor_sync(0xffffffffu, v.x, m);
    v.y = __shfl_xor_sync(0xffffffffu, v.y, m);
    v.z = __shfl_xor_sync(0xffffffffu, v.z, m);
    v.w = __shfl_xor_sync(0xffffffffu, v.w, m);
    return v;
}

// thread = query row (TMEM lane); warp w takes lane quadrant w % 4 and key
// columns [64 (w / 4), 64 (w / 4) + 64) of each tile.
template <int D>
__device__ void q_elementwise(BwQSync &sy, uint32_t tmem, const BwGrid &g, int32_t *status) {
    using Q = BwQShape<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int col0 = 64 * half;                  // this warp's 64 key columns
    int u = 0, ac = 0;
    bool ok = true;
    // this row's log-sum-exp and Delta, fetched one item ahead
    auto fetch = [&](int w, float &l2, float &dl) {
        int b, h, i;
        q_item(w, g, b, h, i);
        const int qrow = i * 128 + r;
        const size_t off = ((size_t)b * g.Hq + h) * g.lse_stride + qrow;
        l2 = qrow < g.T ? g.lse[off] * kLog2e : 0.f;
        dl = qrow < g.T ? g.delta[off] : 0.f;
    };
    // Drain item (b, h, i)'s dQ: called after the next item's first key tile, so
    // the wait for the last dQ MMA overlaps that tile's work.
    auto drain = [&](int b, int h, int i) -> bool {
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(A(sy.acc_full), ac & 1))) return false;
        ++ac;
        ptx::tc_fence_after();
        // Each lane holds 64 bytes of its own row per 32 columns.  A 4 x 4 transpose
        // of 16-byte pieces within each group of four lanes gives lane 4m + p piece p
        // of rows 4m .. 4m + 3, so one store writes 64 contiguous bytes of eight rows
        // (instead of 16 bytes of 32 rows).
        const int p = lane & 3;
        const int row_q = i * 128 + quad * 32 + (lane & ~3);   // the group's first row
        for (int c = half; c < D / 32; c += 2) {
            uint32_t a[32];
            ptx::tmem_ld32(lane_addr + Q::kColAcc + 32 * c, a);
            ptx::tmem_wait_ld();
            uint4 x[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                x[e] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * e]) * g.scale, __uint_as_float(a[8 * e + 1]) * g.scale),
                                  pack_bf16x2(__uint_as_float(a[8 * e + 2]) * g.scale, __uint_as_float(a[8 * e + 3]) * g.scale),
                                  pack_bf16x2(__uint_as_float(a[8 * e + 4]) * g.scale, __uint_as_float(a[8 * e + 5]) * g.scale),
                                  pack_bf16x2(__uint_as_float(a[8 * e + 6]) * g.scale, __uint_as_float(a[8 * e + 7]) * g.scale));
            // stage 1 (lanes p, p ^ 1): slot 2a + r holds piece 2a + (p & 1) of row (p & 2) | r
#pragma unroll
            for (int pr = 0; pr < 4; pr += 2) {
                const bool odd = p & 1;
                const uint4 snd = odd ? x[pr] : x[pr + 1];
                const uint4 rcv = shfl_xor_u4(snd, 1);
                if (odd) x[pr] = rcv; else x[pr + 1] = rcv;
            }
            // stage 2 (lanes p, p ^ 2): slot s holds piece p of row s
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const bool hi = p & 2;
                const uint4 snd = hi ? x[r] : x[2 + r];
                const uint4 rcv = shfl_xor_u4(snd, 2);
                if (hi) x[r] = rcv; else x[2 + r] = rcv;
            }
#pragma unroll
            for (int s2 = 0; s2 < 4; ++s2) {
                const int row = row_q + s2;
                if (row < g.T)
                    *reinterpret_cast<uint4 *>(g.d0 + (((size_t)b * g.T + row) * g.Hq + h) * D + 32 * c + 8 * p) = x[s2];
            }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(A(sy.acc_empty));
        return true;
    };
    float nl2 = 0.f, ndl = 0.f;
    int pb = 0, ph = 0, pi = 0;                 // the previous item
    if (bw_w(0) < g.n_items) fetch(bw_w(0), nl2, ndl);
    for (int kk = 0, w = bw_w(0); w < g.n_items && ok; w = bw_w(++kk)) {
        int b, h, i;
        q_item(w, g, b, h, i);
        const float lse2 = nl2, dlt = ndl;
        if (bw_w(kk + 1) < g.n_items) fetch(bw_w(kk + 1), nl2, ndl);
        const int qrow = i * 128 + r;
        for (int j = 0; j <= i && ok; ++j, ++u) {
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.s_full[u & 1]), (u >> 1) & 1) &&
                                             ptx::mbar_wait(A(sy.dp_full), u & 1));
            if (!ok) break;
            ptx::tc_fence_after();
            const uint32_t sbuf = lane_addr + 128 * (u & 1);
            uint32_t sv[64], dv[64];
            ptx::tmem_ld32(sbuf + col0, *reinterpret_cast<uint32_t(*)[32]>(sv));
            ptx::tmem_ld32(sbuf + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
            ptx::tmem_ld32(lane_addr + Q::kColDP + col0, *reinterpret_cast<uint32_t(*)[32]>(dv));
            ptx::tmem_ld32(lane_addr + Q::kColDP + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(dv + 32));
            ptx::tmem_wait_ld();
            // dP is in registers: the next dP may overwrite it
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(A(sy.dp_free));
            uint32_t dd[32];
            if (j == i)
                q_block<true>(sv, dv, j * 128 + col0, qrow, g.scale_log2, lse2, dlt, dd);
            else
                q_block<false>(sv, dv, j * 128 + col0, qrow, g.scale_log2, lse2, dlt, dd);
            ptx::tmem_st16(sbuf + 32 + col0 / 2, *reinterpret_cast<uint32_t(*)[16]>(dd));
            ptx::tmem_st16(sbuf + 32 + col0 / 2 + 16, *reinterpret_cast<uint32_t(*)[16]>(dd + 16));
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(A(sy.ds_full[u & 1]));
            if (j == 0 && kk > 0) ok = drain(pb, ph, pi);
        }
        if (!ok) break;
        pb = b;
        ph = h;
        pi = i;
    }
    if (ok && bw_w(0) < g.n_items) ok = drain(pb, ph, pi);
    if (!ok && lane == 0) report(status, GQA_DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
// the two tensor-core kernels
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bw_setup(BwSync &sy) {
    if (threadIdx.x == 0) {
        ptx::mbar_init(A(sy.fixed_full), 1);
        ptx::mbar_init(A(sy.fixed_empty), 1);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(A(sy.st_full[s]), 1);
            ptx::mbar_init(A(sy.st_empty[s]), 1);
        }
        ptx::mbar_init(A(sy.acc_full), 1);
        ptx::mbar_init(A(sy.acc_empty), kEwWarps);
        for (int h = 0; h < 2; ++h) {
            ptx::mbar_init(A(sy.h_full[h]), 1);
            ptx::mbar_init(A(sy.h_done[h]), kEwWarps);
        }
        ptx::mbar_init(A(sy.mma_done), 1);
        ptx::fence_barrier_init();
    }
    if ((threadIdx.x >> 5) == kBwMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(&sy.tmem_base), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
}

__device__ __forceinline__ void bw_teardown(BwSync &sy) {
    ptx::tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == kBwMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(sy.tmem_base, 512);
    }
}

template <int D>
__global__ void __launch_bounds__(kBwThreads, 1)
bwd_kv_kernel(const __grid_constant__ BwMaps maps, BwGrid g, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ BwSync sy;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    bw_setup(sy);
    // Delta (and the forward's outputs) come from the kernels before this one.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Delta is complete: the dQ kernel, which reads nothing this kernel writes,
    // may start on the SMs this kernel's CTAs free.
    asm volatile("griddepcontrol.launch_dependents;");
    const uint32_t tmem = sy.tmem_base;
    if (warp >= kEwWarps) {
        ptx::regs_dec<kBwCtlRegs>();
        if (warp == kBwTmaWarp) {
            if (lane == 0) kv_producer<D>(maps, sy, smem, g, status);
            __syncwarp();
        } else if (warp == kBwMmaWarp) {
            kv_mma<D>(sy, smem, tmem, g, status);   // the whole warp
            __syncwarp();
        }
    } else {
        ptx::regs_inc<kBwEwRegs>();
        kv_elementwise<D>(maps, sy, smem, tmem, g, status);
    }
    bw_teardown(sy);
}

__device__ __forceinline__ void bwq_setup(BwQSync &sy) {
    if (threadIdx.x == 0) {
        ptx::mbar_init(A(sy.fixed_full), 1);
        ptx::mbar_init(A(sy.fixed_empty), 1);
        for (int s = 0; s < 3; ++s) {
            ptx::mbar_init(A(sy.k_full[s]), 1);
            ptx::mbar_init(A(sy.k_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(A(sy.v_full[s]), 1);
            ptx::mbar_init(A(sy.v_empty[s]), 1);
            ptx::mbar_init(A(sy.s_full[s]), 1);
            ptx::mbar_init(A(sy.ds_full[s]), kEwWarps);   // one elected lane per elementwise warp
        }
        ptx::mbar_init(A(sy.dp_full), 1);
        ptx::mbar_init(A(sy.dp_free), kEwWarps);
        ptx::mbar_init(A(sy.acc_full), 1);
        ptx::mbar_init(A(sy.acc_empty), kEwWarps);
        ptx::mbar_init(A(sy.mma_done), 1);
        ptx::fence_barrier_init();
    }
    if ((threadIdx.x >> 5) == kBwMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(&sy.tmem_base), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
}

template <int D>
__global__ void __launch_bounds__(kBwThreads, 1)
bwd_q_kernel(const __grid_constant__ BwMaps maps, BwGrid g, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ BwQSync sy;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    bwq_setup(sy);
    const uint32_t tmem = sy.tmem_base;
    if (warp >= kEwWarps) {
        ptx::regs_dec<kBwCtlRegs>();
        if (warp == kBwTmaWarp) {
            if (lane == 0) q_producer<D>(maps, sy, smem, g, status);
            __syncwarp();
        } else if (warp == kBwMmaWarp) {
            q_mma<D>(sy, smem, tmem, g, status);   // the whole warp
            __syncwarp();
        }
    } else {
        ptx::regs_inc<kBwEwRegs>();
        q_elementwise<D>(sy, tmem, g, status);
    }
    // Launched once every dK/dV CTA had seen Delta complete (no wait needed at the
    // start); wait for the dK/dV kernel here, so this launch's end means both are
    // done for whatever the stream runs next.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kBwMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(sy.tmem_base, 512);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int lse_stride_of(int T) { return (T + 3) & ~3; }

template <typename K>
cudaError_t launch_pdl(K kern, dim3 grid, dim3 block, int smem, cudaStream_t s,
                       const BwMaps &maps, const BwGrid &g, int32_t *status) {
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, maps, g, status);
}

template <int D>
gqa_status launch_backward(const void *q, const void *k, const void *v, const void *out,
                           const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                           int T, int Hq, int Hkv, int Lmax, float scale, float *delta,
                           int32_t *status, cudaStream_t s) {
    using S = BwShape<D>;
    const int ls = lse_stride_of(T);
    float *nl2 = delta + (size_t)B * Hq * ls;         // -lse log2(e), written with Delta
    BwMaps maps;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T, (cuuint64_t)B};
        const cuuint64_t str[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2,
                                   (cuuint64_t)T * Hq * D * 2};
        const cuuint32_t box[4] = {64, 1, 128, 1};
        if (!encode(&maps.q, q, 4, dims, str, box)) return GQA_ERR_CUDA;
        if (!encode(&maps.dout, dout, 4, dims, str, box)) return GQA_ERR_CUDA;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)B * Hkv};
        const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)Lmax * D * 2};
        const cuuint32_t box[3] = {64, 128, 1};
        if (!encode(&maps.k, k, 3, dims, str, box)) return GQA_ERR_CUDA;
        if (!encode(&maps.v, v, 3, dims, str, box)) return GQA_ERR_CUDA;
        if (!encode(&maps.dk, dk, 3, dims, str, box)) return GQA_ERR_CUDA;
        if (!encode(&maps.dv, dv, 3, dims, str, box)) return GQA_ERR_CUDA;
    }
    if (!encode_f32_2d(&maps.lse, nl2, (cuuint64_t)T, (cuuint64_t)B * Hq, (cuuint64_t)ls * 4, 128))
        return GQA_ERR_CUDA;
    if (!encode_f32_2d(&maps.delta, delta, (cuuint64_t)T, (cuuint64_t)B * Hq, (cuuint64_t)ls * 4,
                       128))
        return GQA_ERR_CUDA;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GQA_ERR_CUDA;
    BwGrid g;
    g.B = B;
    g.T = T;
    g.Hq = Hq;
    g.Hkv = Hkv;
    g.nT = (T + 127) / 128;
    g.lse_stride = ls;
    g.scale = scale;
    g.scale_log2 = scale * kLog2e;
    g.lse = lse;
    g.delta = delta;
    g.Lmax = Lmax;

    // 1. Delta
    {
        cudaLaunchAttribute pdl[1];
        pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pdl[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        const int tpr = D / 8 > 8 ? 16 : 8;
        constexpr int kPasses = 2;             // rows per lane (4 and 8 measured slower)
        const long long per_cta = 256 / tpr * kPasses;
        cfg.gridDim = dim3((unsigned)(((long long)T * Hq + per_cta - 1) / per_cta), (unsigned)B);
        cfg.blockDim = dim3(256);
        cfg.stream = s;
        cfg.attrs = pdl;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, delta_kernel<D, kPasses>, static_cast<const uint16_t *>(out),
                               static_cast<const uint16_t *>(dout), lse, delta, nl2, T, Hq,
                               ls) !=
            cudaSuccess)
            return GQA_ERR_CUDA;
    }
    // The warpgroup register split assumes 168 registers per thread at launch;
    // with any other count the increases could not be met, so refuse.
    {
        cudaFuncAttributes a1, a2;
        if (cudaFuncGetAttributes(&a1, bwd_kv_kernel<D>) != cudaSuccess ||
            cudaFuncGetAttributes(&a2, bwd_q_kernel<D>) != cudaSuccess)
            return GQA_ERR_CUDA;
        if (a1.numRegs != 168 || a2.numRegs != 168) return GQA_ERR_UNSUPPORTED;
    }
    // 2. dK, dV
    {
        auto kern = bwd_kv_kernel<D>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemKV) !=
            cudaSuccess)
            return GQA_ERR_CUDA;
        BwGrid gk = g;
        gk.n_items = g.nT * B * Hkv;
        gk.d0 = static_cast<uint16_t *>(dk);
        gk.d1 = static_cast<uint16_t *>(dv);
        const int grid = gk.n_items < sms ? gk.n_items : sms;
        if (launch_pdl(kern, dim3(grid), dim3(kBwThreads), S::kSmemKV, s, maps, gk, status) !=
            cudaSuccess)
            return GQA_ERR_CUDA;
    }
    // 3. dQ
    {
        auto kern = bwd_q_kernel<D>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 BwQShape<D>::kSmem) != cudaSuccess)
            return GQA_ERR_CUDA;
        BwGrid gq = g;
        gq.n_items = g.nT * B * Hq;
        gq.d0 = static_cast<uint16_t *>(dq);
        gq.d1 = nullptr;
        const int grid = gq.n_items < sms ? gq.n_items : sms;
        if (launch_pdl(kern, dim3(grid), dim3(kBwThreads), BwQShape<D>::kSmem, s, maps, gq, status) !=
            cudaSuccess)
            return GQA_ERR_CUDA;
    }
    return gqa_host::launch_status();
}

}  // namespace
}  // namespace gqa

extern "C" size_t gqa_backward_workspace_bytes(int B, int T, int Hq) {
    if (B < 1 || T < 1 || Hq < 1) return 0;
    return 2 * (size_t)B * Hq * gqa::lse_stride_of(T) * 4;    // Delta, then -lse log2(e)
}

extern "C" gqa_status gqa_attention_backward(const void *q, const void *k, const void *v,
                                             const void *out, const void *dout, const float *lse,
                                             void *dq, void *dk, void *dv, int B, int T, int Hq,
                                             int Hkv, int D, int Lmax, float scale, void *ws,
                                             size_t ws_bytes, int32_t *status_dev, void *stream) {
    using namespace gqa_host;
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || B < 1 || T < 1 ||
        Hq < 1 || Hkv < 1 || Lmax < 1)
        return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return GQA_ERR_INVALID_ARG;
    if (!head_dim_ok(D)) return GQA_ERR_UNSUPPORTED;
    if (Lmax % 128 != 0) return GQA_ERR_INVALID_ARG;
    if (T > Lmax) return GQA_ERR_CAPACITY;
    if ((long long)((T + 127) / 128) * B * Hq > 0x7fffffffLL) return GQA_ERR_INVALID_ARG;
    if ((long long)T * Hq > 0x7fffffffLL || B > 65535) return GQA_ERR_INVALID_ARG;  // Delta's grid
    const size_t need = gqa_backward_workspace_bytes(B, T, Hq);
    if (!ws || ws_bytes < need || !aligned16(ws)) return GQA_ERR_WORKSPACE;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        major != 10)
        return GQA_ERR_UNSUPPORTED;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *delta = static_cast<float *>(ws);          // [B, Hq, lse stride] each
    switch (D) {
        case 64: return gqa::launch_backward<64>(q, k, v, out, dout, lse, dq, dk, dv, B, T, Hq, Hkv, Lmax, sc, delta, status_dev, s);
        case 96: return gqa::launch_backward<96>(q, k, v, out, dout, lse, dq, dk, dv, B, T, Hq, Hkv, Lmax, sc, delta, status_dev, s);
        default: return gqa::launch_backward<128>(q, k, v, out, dout, lse, dq, dk, dv, B, T, Hq, Hkv, Lmax, sc, delta, status_dev, s);
    }
}
