// prefill.cu -- causal GQA prefill on the 5th-generation tensor cores (tcgen05).
//
// out[b,t,h] = sum_{s<=t} softmax_s(q[b,t,h] . K[b,h/g,s] * scale) V[b,h/g,s]:
// the causal scaled_dot_product_attention of page "训练3.8B LLM至0.384 CORE，
// 成本998美元 – Hugo Vergnes" (section "无效的方法"), with query heads sharing
// K/V heads in groups (page "750美元从零训练3个LLM：一位开发者的实战复盘", section
// "V2：引入前沿技术").  Flash-style: the softmax is taken online over key tiles in
// fp32, so the T x T score matrix never exists outside the tensor memory.
//
// One CTA owns two 128-row query tiles of one (b, h) -- rows [256i, 256i+128)
// and [256i+128, 256i+256) -- and streams the key/value tiles they need.
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of tile 0 (thread = query row = TMEM lane), 232 registers
//   warps 4-7  softmax of tile 1, 232 registers
//   warp 8     TMA producer: Q tiles once, then a K ring and a V ring  } 40
//   warp 9     MMA issuer (one thread): S_t = Q_t K^T and O_t += P_t V } registers
//   warps 10-11 idle (they complete the third warpgroup)              }
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) fp32 scores, with the
// bf16 probabilities P_t written over the first 64 columns of S_t; O0 [256, 256+D)
// O1 [384, 384+D) fp32 accumulators.
// The tensor core alternates between the tiles -- PV0(j), S0(j+1), PV1(j),
// S1(j+1) -- so the softmax of one tile runs while the other tile's two MMAs
// execute.  A commit after S_t(j+1) also covers PV_t(j), so the softmax may
// rescale O_t in TMEM as soon as its next scores are ready.  O_t is only
// rescaled when the running maximum grows by more than 2^8 (the stale maximum
// otherwise keeps p <= 256, exact in the final normalisation).
//
// Every mbarrier wait is bounded; a role that times out raises GQA_DEV_TIMEOUT
// and stops, the producer then waits (bounded) for its copies in flight and the
// MMA thread for its MMAs before the tensor memory is released.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace gqa {
namespace {

constexpr int kPfThreads = 384;   // three warpgroups
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
// Registers: launched at 168 per thread (65536 / 384, rounded down to 8); the two
// softmax warpgroups take 224 each and the producer/MMA warpgroup keeps 56:
// 2 * 224 + 56 = 3 * 168, so the increases are exactly covered by the decrease.
constexpr int kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 224;
constexpr uint32_t kControlRegs = 56;
static_assert(2 * kSoftmaxRegs + kControlRegs == 3 * kLaunchRegs, "register split must balance");
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only past 2^8 growth

template <int D>
struct PfShape {
    static constexpr int kBlocks = (D + 63) / 64;           // 128-byte column blocks
    static constexpr int kBlockBytes = 128 * 128;           // 128 rows x 128 bytes
    static constexpr int kTileBytes = kBlocks * kBlockBytes;
    static constexpr int kStages = D == 64 ? 4 : 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kSmem = kOffV + kStages * kTileBytes + 1024;   // + 1 KB alignment slack
    static constexpr int kKSteps = D / 16;
};

struct PfMaps {
    CUtensorMap q, k, v;
};

struct PfSync {
    uint64_t q_full;
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    uint64_t s_full[2], p_full[2], o_final[2];
    uint64_t mma_done;
    uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t A(const uint64_t &b) { return ptx::smem_addr(&b); }

template <int D>
__device__ void producer(const PfMaps &maps, PfSync &sy, uint8_t *smem, int b, int h, int kvh,
                         int Hkv, int q0, bool has1, int n_kv, int32_t *status) {
    using S = PfShape<D>;
    // The kernel is a programmatic dependent of the preceding one (normally the
    // append that rotated q and filled the cache): wait for it before loading.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t qbytes = S::kTileBytes * (has1 ? 2 : 1);
    ptx::mbar_arrive_expect_tx(A(sy.q_full), qbytes);
    for (int t = 0; t < (has1 ? 2 : 1); ++t)
        for (int kb = 0; kb < S::kBlocks; ++kb)
            ptx::tma_load_4d(ptx::smem_addr(smem + S::kOffQ + t * S::kTileBytes + kb * S::kBlockBytes),
                             &maps.q, A(sy.q_full), kb * 64, h, q0 + 128 * t, b);
    int issued_k = 0, issued_v = 0;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % S::kStages;
        const uint32_t par = ((j / S::kStages) & 1) ^ 1;
        ok = ptx::mbar_wait(A(sy.k_empty[st]), par);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(A(sy.k_full[st]), S::kTileBytes);
        for (int kb = 0; kb < S::kBlocks; ++kb)
            ptx::tma_load_3d(ptx::smem_addr(smem + S::kOffK + st * S::kTileBytes + kb * S::kBlockBytes),
                             &maps.k, A(sy.k_full[st]), kb * 64, j * 128, b * Hkv + kvh);
        issued_k = j + 1;
        ok = ptx::mbar_wait(A(sy.v_empty[st]), par);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(A(sy.v_full[st]), S::kTileBytes);
        for (int kb = 0; kb < S::kBlocks; ++kb)
            ptx::tma_load_3d(ptx::smem_addr(smem + S::kOffV + st * S::kTileBytes + kb * S::kBlockBytes),
                             &maps.v, A(sy.v_full[st]), kb * 64, j * 128, b * Hkv + kvh);
        issued_v = j + 1;
    }
    if (!ok) {
        report(status, GQA_DEV_TIMEOUT);
        // Let every copy already issued land before the CTA can retire.
        ptx::mbar_wait(A(sy.q_full), 0);
        for (int j = (issued_k > S::kStages ? issued_k - S::kStages : 0); j < issued_k; ++j)
            ptx::mbar_wait(A(sy.k_full[j % S::kStages]), (j / S::kStages) & 1);
        for (int j = (issued_v > S::kStages ? issued_v - S::kStages : 0); j < issued_v; ++j)
            ptx::mbar_wait(A(sy.v_full[j % S::kStages]), (j / S::kStages) & 1);
    }
}

template <int D>
__device__ void mma_issuer(PfSync &sy, uint8_t *smem, uint32_t tmem, bool has1, int n0, int n1,
                           int n_kv, int32_t *status) {
    using S = PfShape<D>;
    constexpr uint32_t idS = ptx::idesc_bf16_f32(128, 128, false);
    constexpr uint32_t idO = ptx::idesc_bf16_f32(128, D, true);
    const uint32_t q_base = ptx::smem_addr(smem + S::kOffQ);
    const uint32_t k_base = ptx::smem_addr(smem + S::kOffK);
    const uint32_t v_base = ptx::smem_addr(smem + S::kOffV);

    auto issue_s = [&](int t, int j) {
        const uint32_t qa = q_base + t * S::kTileBytes;
        const uint32_t ka = k_base + (j % S::kStages) * S::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < S::kKSteps; ++ks) {
            const uint32_t off = (ks >> 2) * S::kBlockBytes + (ks & 3) * 32;
            ptx::mma_ss(tmem + t * 128, ptx::smem_desc_sw128(qa + off, 16, 1024),
                        ptx::smem_desc_sw128(ka + off, 16, 1024), idS, ks > 0);
        }
        ptx::mma_commit(A(sy.s_full[t]));
    };
    auto issue_pv = [&](int t, int j) {
        const uint32_t va = v_base + (j % S::kStages) * S::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            ptx::mma_ts(tmem + 256 + t * 128, tmem + t * 128 + ks * 8,
                        ptx::smem_desc_sw128(va + ks * 2048, S::kBlockBytes, 1024), idO,
                        (j > 0 || ks > 0) ? 1u : 0u);
    };

    bool ok = ptx::mbar_wait(A(sy.q_full), 0) && ptx::mbar_wait(A(sy.k_full[0]), 0);
    if (ok) {
        ptx::tc_fence_after();
        issue_s(0, 0);
        if (has1) issue_s(1, 0);
        ptx::mma_commit(A(sy.k_empty[0]));
    }
    for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % S::kStages;
        ok = ptx::mbar_wait(A(sy.v_full[st]), (j / S::kStages) & 1);
        if (!ok) break;
        const int jn = j + 1;
        const int stn = jn % S::kStages;
        bool k_next = false;
        if (j < n0) {
            ok = ptx::mbar_wait(A(sy.p_full[0]), j & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_pv(0, j);
            if (jn < n0) {
                ok = ptx::mbar_wait(A(sy.k_full[stn]), (jn / S::kStages) & 1);
                if (!ok) break;
                k_next = true;
                issue_s(0, jn);
            } else {
                ptx::mma_commit(A(sy.o_final[0]));
            }
        }
        if (has1 && j < n1) {
            ok = ptx::mbar_wait(A(sy.p_full[1]), j & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            issue_pv(1, j);
            if (jn < n1) {
                if (!k_next) {
                    ok = ptx::mbar_wait(A(sy.k_full[stn]), (jn / S::kStages) & 1);
                    if (!ok) break;
                    k_next = true;
                }
                issue_s(1, jn);
            } else {
                ptx::mma_commit(A(sy.o_final[1]));
            }
        }
        ptx::mma_commit(A(sy.v_empty[st]));
        if (k_next) ptx::mma_commit(A(sy.k_empty[stn]));
    }
    if (!ok) report(status, GQA_DEV_TIMEOUT);
    // No MMA may still be writing tensor memory when it is released.
    ptx::mma_commit(A(sy.mma_done));
    ptx::mbar_wait(A(sy.mma_done), 0);
}

template <int D>
__device__ void softmax_tile(PfSync &sy, uint32_t tmem, int t, int q_first, int nt, int T,
                             float scale_log2, uint16_t *out_row_base, size_t row_stride,
                             int32_t *status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = (warp & 3) * 32 + lane;
    const int qrow = q_first + row;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = t * 128, o_col = 256 + t * 128;
    const int diag = q_first / 128;

    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.s_full[t]), j & 1));
        if (!ok) break;
        ptx::tc_fence_after();
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(lane_addr + s_col + 32 * c, sv[c]);
        ptx::tmem_wait_ld();
#define SV(c) __uint_as_float(sv[(c) >> 5][(c) & 31])

        const int key0 = j * 128;
        if (j == diag || key0 + 128 > T) {
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                const int key = key0 + c;
                if (key > qrow || key >= T) sv[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
        }
        // Row maximum: four independent chains of three-input max.
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
            mx0 = ptx::fmax3(mx0, SV(c), SV(c + 1));
            mx1 = ptx::fmax3(mx1, SV(c + 2), SV(c + 3));
            mx2 = ptx::fmax3(mx2, SV(c + 4), SV(c + 5));
            mx3 = ptx::fmax3(mx3, SV(c + 6), SV(c + 7));
        }
        const float smax = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const float m_new = fmaxf(m, smax * scale_log2);
        const bool resc = m_new > m + kRescaleThreshold;
        const float alpha = resc ? ex2(m - m_new) : 1.f;
        if (resc) {
            l *= alpha;
            m = m_new;
        }
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(lane_addr + o_col + 32 * c, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                ptx::tmem_st32(lane_addr + o_col + 32 * c, o);
            }
        }
        // p = 2^(s * scale_log2 - m): packed FMA for the exponent argument, the
        // special-function unit for 2^x, four independent partial row sums.
        const float neg_m = -m;
        float la0 = 0.f, la1 = 0.f, lb0 = 0.f, lb1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t p[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float x0, x1;
                ptx::ffma2(x0, x1, SV(32 * c + 2 * e), SV(32 * c + 2 * e + 1), scale_log2,
                           scale_log2, neg_m, neg_m);
                const float p0 = ex2(x0), p1 = ex2(x1);
                p[e] = pack_bf16x2(p0, p1);
                if (e & 1)
                    ptx::fadd2(la0, la1, la0, la1, p0, p1);
                else
                    ptx::fadd2(lb0, lb1, lb0, lb1, p0, p1);
            }
            ptx::tmem_st16(lane_addr + s_col + 16 * c, p);
        }
#undef SV
        l += (la0 + la1) + (lb0 + lb1);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(A(sy.p_full[t]));
    }
    if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.o_final[t]), 0));
    if (!ok) {
        if (lane == 0) report(status, GQA_DEV_TIMEOUT);
        return;
    }
    ptx::tc_fence_after();
    const float inv_l = 1.f / l;
    uint16_t *dst = out_row_base + (size_t)qrow * row_stride;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        ptx::tmem_ld32(lane_addr + o_col + 32 * c, o);
        ptx::tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (qrow < T) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c);
            d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
            d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
            d4[2] = make_uint4(w[8], w[9], w[10], w[11]);
            d4[3] = make_uint4(w[12], w[13], w[14], w[15]);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const __grid_constant__ PfMaps maps, uint16_t *__restrict__ out, int B, int T,
               int Hq, int Hkv, float scale_log2, int n_pairs, int32_t *status) {
    using S = PfShape<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ PfSync sy;

    // Longest query pairs first; the heads of one KV group run side by side.
    const int per_pair = Hq * B;
    const int pair = n_pairs - 1 - (int)(blockIdx.x / per_pair);
    const int rest = (int)(blockIdx.x % per_pair);
    const int h = rest % Hq, b = rest / Hq;
    const int kvh = h / (Hq / Hkv);
    const int q0 = pair * 256;
    const bool has1 = q0 + 128 < T;
    const int n0 = (min(T, q0 + 128) + 127) / 128;
    const int n1 = has1 ? (min(T, q0 + 256) + 127) / 128 : 0;
    const int n_kv = has1 ? n1 : n0;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        ptx::mbar_init(A(sy.q_full), 1);
        for (int i = 0; i < S::kStages; ++i) {
            ptx::mbar_init(A(sy.k_full[i]), 1);
            ptx::mbar_init(A(sy.k_empty[i]), 1);
            ptx::mbar_init(A(sy.v_full[i]), 1);
            ptx::mbar_init(A(sy.v_empty[i]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(A(sy.s_full[t]), 1);
            ptx::mbar_init(A(sy.p_full[t]), 4);   // one elected lane per softmax warp
            ptx::mbar_init(A(sy.o_final[t]), 1);
        }
        ptx::mbar_init(A(sy.mma_done), 1);
        ptx::fence_barrier_init();
    }
    if (warp == kTmaWarp && lane == 0) {
        ptx::prefetch_tensormap(&maps.q);
        ptx::prefetch_tensormap(&maps.k);
        ptx::prefetch_tensormap(&maps.v);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(&sy.tmem_base), 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sy.tmem_base;

    if (warp >= 8) {
        ptx::regs_dec<kControlRegs>();
        if (warp == kTmaWarp) {
            if (lane == 0) producer<D>(maps, sy, smem, b, h, kvh, Hkv, q0, has1, n_kv, status);
            __syncwarp();
        } else if (warp == kMmaWarp) {
            if (lane == 0) mma_issuer<D>(sy, smem, tmem, has1, n0, n1, n_kv, status);
            __syncwarp();
        }
    } else {
        ptx::regs_inc<kSoftmaxRegs>();
        const int t = warp >> 2;
        if (t == 0 || has1) {
            uint16_t *base = out + ((size_t)b * T * Hq + h) * D;
            softmax_tile<D>(sy, tmem, t, q0 + 128 * t, t == 0 ? n0 : n1, T, scale_log2, base,
                            (size_t)Hq * D, status);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor map with 128-byte swizzle and a {64, rows...} box; OOB reads are zero.
bool encode(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
            const cuuint64_t *strides, const cuuint32_t *box) {
    EncodeTiledFn fn = encoder();
    if (!fn) return false;
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
gqa_status launch_prefill(const void *q, const void *kc, const void *vc, void *out, int B, int T,
                          int Hq, int Hkv, int Lmax, float scale_log2, int32_t *status,
                          cudaStream_t s) {
    using S = PfShape<D>;
    PfMaps maps;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T, (cuuint64_t)B};
        const cuuint64_t str[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2,
                                   (cuuint64_t)T * Hq * D * 2};
        const cuuint32_t box[4] = {64, 1, 128, 1};
        if (!encode(&maps.q, q, 4, dims, str, box)) return GQA_ERR_CUDA;
    }
    {
        // Rows beyond T are outside the map, so the copies zero-fill them and
        // the unused cache slots (whatever they hold) are never read.
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)B * Hkv};
        const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)Lmax * D * 2};
        const cuuint32_t box[3] = {64, 128, 1};
        if (!encode(&maps.k, kc, 3, dims, str, box)) return GQA_ERR_CUDA;
        if (!encode(&maps.v, vc, 3, dims, str, box)) return GQA_ERR_CUDA;
    }
    auto kern = prefill_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem) !=
        cudaSuccess)
        return GQA_ERR_CUDA;
    // The warpgroup register split assumes the launch allocation of kLaunchRegs per
    // thread; with any other count the increases could not be satisfied, so refuse.
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return GQA_ERR_CUDA;
    if (attr.numRegs != kLaunchRegs) return GQA_ERR_UNSUPPORTED;
    const int n_pairs = (T + 255) / 256;
    const long long grid = (long long)n_pairs * Hq * B;
    // Programmatic dependent launch: the prologue (barriers, tensor memory,
    // descriptor prefetch) overlaps the tail of the preceding kernel; the TMA
    // producer waits for that kernel before its first load.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = S::kSmem;
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, maps, static_cast<uint16_t *>(out), B, T, Hq, Hkv,
                           scale_log2, n_pairs, status) != cudaSuccess)
        return GQA_ERR_CUDA;
    return gqa_host::launch_status();
}

bool device_is_sm100() {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return false;
    return major == 10;
}

}  // namespace
}  // namespace gqa

extern "C" gqa_status gqa_prefill(const void *q, const void *k_cache, const void *v_cache,
                                  void *out, int B, int T, int Hq, int Hkv, int D, int Lmax,
                                  float scale, int32_t *status_dev, void *stream) {
    using namespace gqa_host;
    if (!q || !k_cache || !v_cache || !out || B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Lmax < 1)
        return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return GQA_ERR_INVALID_ARG;
    if (!head_dim_ok(D)) return GQA_ERR_UNSUPPORTED;
    if (Lmax % 128 != 0) return GQA_ERR_INVALID_ARG;
    if (T > Lmax) return GQA_ERR_CAPACITY;
    if ((long long)((T + 255) / 256) * Hq * B > 0x7fffffffLL) return GQA_ERR_INVALID_ARG;
    if (!gqa::device_is_sm100()) return GQA_ERR_UNSUPPORTED;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
    const float sl2 = sc * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (D) {
        case 64: return gqa::launch_prefill<64>(q, k_cache, v_cache, out, B, T, Hq, Hkv, Lmax, sl2, status_dev, s);
        case 96: return gqa::launch_prefill<96>(q, k_cache, v_cache, out, B, T, Hq, Hkv, Lmax, sl2, status_dev, s);
        default: return gqa::launch_prefill<128>(q, k_cache, v_cache, out, B, T, Hq, Hkv, Lmax, sl2, status_dev, s);
    }
}
