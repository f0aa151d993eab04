// prefill.cu -- causal GQA prefill on the 5th-generation tensor cores (tcgen05).
//
// out[b,t,h] = sum_{s<=p(t)} softmax_s(q[b,t,h] . K[b,h/g,s] * scale) V[b,h/g,s]
// with p(t) = pos0[b] + t: the causal scaled_dot_product_attention of page
// "训练3.8B LLM至0.384 CORE，成本998美元 – Hugo Vergnes" (section "无效的方法"),
// with query heads sharing K/V heads in groups (page "750美元从零训练3个LLM：一位
// 开发者的实战复盘", section "V2：引入前沿技术").  pos0 = 0 is a prompt prefill;
// pos0 > 0 continues a cached prefix (the new tokens attend to the cache and to
// each other causally, page "750美元从零训练3个LLM", section "V3：扩容与推理优化").
// Flash-style: the softmax is taken online over key tiles in fp32, so the score
// matrix never exists outside the tensor memory.
//
// Persistent: one CTA per SM takes items one after another; an item is two
// 128-row query tiles that share a KV head, and streams the key/value tiles
// they need.  The (query tile, head) tiles of one (b, KV head) are listed tile
// by tile, the group's query heads within a tile, and taken two at a time: with
// grouped heads most items are one query tile of two heads, whose key ranges
// are the same, and the rest two consecutive tiles (for documents this cut the
// steps where one tile waits on the other by half: 143 -> 139 us on the packed
// 8 x 2048 prompt).  Items are numbered longest first and, with four or more per
// CTA, taken from a launch-wide counter as CTAs free up (else dealt statically).
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of tile 0 (thread = query row = TMEM lane), 216 registers
//   warps 4-7  softmax of tile 1, 216 registers
//   warp 8     TMA producer: Q tiles, then a K ring and a V ring    } 72
//   warp 9     MMA issuer: S_t = Q_t K^T, O_t += P_t V (one elected } registers
//              lane issues; the whole warp runs the loop)           }
//   warps 10-11 idle (they complete the third warpgroup)            }
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) fp32 scores, with the
// bf16 probabilities P_t written over the first 64 columns of S_t; O0 [256, 256+D)
// O1 [384, 384+D) fp32 accumulators.
// The tensor core alternates between the tiles -- PV0(j), S0(j+1), PV1(j),
// S1(j+1) -- so the softmax of one tile runs while the other tile's two MMAs
// execute.  The softmax hands P over in two halves (key columns
// 0-63, then 64-127) and the first half's P V product runs while it computes
// the second half.  A commit after S_t(j+1) also covers PV_t(j), so the softmax may
// rescale O_t in TMEM as soon as its next scores are ready.  O_t is only
// rescaled when the running maximum grows by more than 2^8 (the stale maximum
// otherwise keeps p <= 256, exact in the final normalisation).
// The output leaves through shared memory: a softmax group normalises O_t 64
// columns at a time into its 16 KB staging (128-byte swizzle) and one of its
// threads stores the block with the output's tensor map (whole lines; storing
// each thread's row straight from registers writes 16 bytes of 32 rows per
// instruction and cost 10 % of the prompt kernel).  Tiles with rows past the
// sequence's end (the ragged last tile, chunks) store their valid rows directly.
//
// Documents packed into one sequence (page "训练3.8B LLM…", section "无效的方法":
// masking at document boundaries, flex-attention style): query t sees only keys
// doc_start[t] .. t.  Each query tile starts at the key tile holding its first
// row's doc_start, so tiles wholly before a document are never loaded, and the
// scores below a row's own start are masked.
//
// Continuation chunks read the cache up to slot pos0 + n_tok - 1 (the last
// valid key); slots past it in the item's last key tile may hold anything,
// NaN included.  Their scores are masked, and before the last P . V product
// the softmax group that owns it zeroes those rows of the V tile in shared
// memory, so a zero probability never meets a NaN value.  (A prompt prefill
// needs neither: its tensor maps end at row T and the copies zero-fill.)
//
// Every mbarrier wait is bounded; a role that times out raises GQA_DEV_TIMEOUT
// and stops, the producer then waits (bounded) for its copies in flight and the
// MMA thread for its MMAs before the tensor memory is released.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace gqa {
namespace {

constexpr int kPfThreads = 384;   // three warpgroups
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
// Registers: launched at 168 per thread (65536 / 384, rounded down to 8); the two
// softmax warpgroups take 216 each and the producer/MMA warpgroup keeps 72:
// 2 * 216 + 72 = 3 * 168, so the increases are exactly covered by the decrease.
// (At 208 / 88 the softmax spilled about 140 bytes per thread; 216 leaves it
// 60 bytes in the chunk mode and none elsewhere: chunks 164 -> 158 us,
// documents 140 -> 138 us, the prompt 1 us faster, outputs bit-identical.)
constexpr int kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 216;
constexpr uint32_t kControlRegs = 72;
static_assert(2 * kSoftmaxRegs + kControlRegs == 3 * kLaunchRegs, "register split must balance");
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only past 2^8 growth

template <int D>
struct PfShape {
    static constexpr int kBlocks = (D + 63) / 64;           // 128-byte column blocks
    static constexpr int kBlockBytes = 128 * 128;           // 128 rows x 128 bytes
    static constexpr int kTileBytes = kBlocks * kBlockBytes;
    // K and V rings next to the two Q tiles and the output staging (D = 128:
    // K 2 + V 2 stages of 32 KB; D = 64: 4 + 4 of 16 KB); the staging holds one
    // 64-column block of an output tile per softmax group (2 x 16 KB).
    static constexpr int kStagesK = D == 64 ? 4 : 2;
    static constexpr int kStagesV = D == 64 ? 4 : 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kStagesK * kTileBytes;
    static constexpr int kOffO = kOffV + kStagesV * kTileBytes;
    static constexpr int kSmem = kOffO + 2 * kBlockBytes + 1024;   // + 1 KB alignment slack
    static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
    static constexpr int kKSteps = D / 16;
};

struct PfMaps {
    CUtensorMap q, k, v, o;
};

struct PfSync {
    uint64_t item_full[4], item_empty[4];   // the CTA's item ring (producer -> the other roles)
    int item[4][16];                        // item number (-1: no more), then its PfItem
    uint64_t q_full, q_empty;
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    uint64_t s_full[2], p_half[2], p_full[2], o_final[2];
    uint64_t mma_done;
    uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t A(const uint64_t &b) { return ptx::smem_addr(&b); }

// Work item w of the grid's items: two query tiles (tile, head) of one sequence
// and KV head.  Items are numbered longest first (pairs nearer the end of the
// chunk see more keys), with the (b, KV head) pairs of one rank side by side.
// Kernel modes: a prompt from position 0, a continuation chunk after a cached
// prefix, a prompt of packed documents, or a prompt that also stores each row's
// log-sum-exp for the backward.
constexpr int kPrompt = 0, kChunkMode = 1, kDocs = 2, kPromptLse = 3;

struct PfItem {
    int b, h, kvh, q0, n0, n1, n_kv;   // tile 0: head h, rows [q0, q0 + 128)
    int h1, q1;        // tile 1: head h1, rows [q1, q1 + 128) (q1 = q0 or q0 + 128)
    int lo0, lo1;      // first key tile of each query tile (documents; else 0)
    int P, N;          // first position of the chunk, valid new tokens (0: no work)
    int r_valid;       // valid key rows in the last key tile (128: the tile is full)
    bool has1;
};

struct PfGrid {
    int n_items, n_pairs, B, T, Hq, Hkv, Lmax;
    int *work;                     // the launch's item counter (items handed out so far)
    const int32_t *pos0, *n_tok;   // chunk positions / token counts (NULL: 0 / T)
    const int32_t *doc_start;      // [B, T] first position of each token's document
    float *lse;                    // optional [B, Hq, lse_stride] row log-sum-exp (prompts)
    int lse_stride;
};

// Items are dealt out dynamically: the producer takes the next item number from
// the launch's counter when it starts loading that item, i.e. once it has issued
// every load of the item before (items are numbered longest first, so this is
// greedy longest-first scheduling), reads the item's sequence data, decodes
// the item and passes it to the CTA's other roles through a four-slot ring in
// shared memory.
// (Static dealing left the CTAs' finish times max/mean 1.05 apart on a prompt
// and 1.17 on documents and chunks.)  Item number -1 marks the end.
constexpr int kItemReaders = 9;        // the 8 softmax warps and the MMA warp

// Static dealing, for launches with few items per CTA: the k-th item of this CTA,
// dealt out in rounds of gridDim.x; a prompt's rounds alternate direction (snake
// order) so that a CTA drawing a long item in one round draws a short one next.
template <int kMode>
__device__ __forceinline__ int pf_static_w(int k) {
    const int G = gridDim.x, c = blockIdx.x;
    constexpr bool snake = kMode == kPrompt || kMode == kPromptLse;
    return k * G + ((snake && (k & 1)) ? G - 1 - c : c);
}
// Item counters: a launch takes one slot (round robin on the host), its CTAs
// count themselves out in g_pf_done and the last one zeroes both, so the slot
// is clean for the launch that next takes it (launches in flight at once take
// different slots).
constexpr int kWorkSlots = 256;
__device__ int g_pf_work[kWorkSlots];
__device__ unsigned g_pf_done[kWorkSlots];


// Item w's tiles: entries 2p and 2p + 1 (p = n_pairs - 1 - rank, longest first)
// of its (b, KV head)'s list of (query tile, head), tile by tile and the G
// query heads of the group within a tile; an odd list leaves the last item one
// tile.
struct PfTiles {
    int b, kvh, h0, q0, h1, q1;
    bool has1;
};
__device__ __forceinline__ PfTiles pf_tiles(int w, const PfGrid &g) {
    const int per = g.B * g.Hkv, G = g.Hq / g.Hkv, nT = (g.T + 127) / 128;
    const int rank = w / per, rest = w - rank * per;
    PfTiles x;
    x.b = rest / g.Hkv;
    x.kvh = rest - x.b * g.Hkv;
    const int e0 = 2 * (g.n_pairs - 1 - rank), e1 = e0 + 1;
    x.q0 = (e0 / G) * 128;
    x.h0 = x.kvh * G + e0 % G;
    x.has1 = e1 < nT * G;
    x.q1 = x.has1 ? (e1 / G) * 128 : x.q0;
    x.h1 = x.has1 ? x.kvh * G + e1 % G : x.h0;
    return x;
}

// What an item needs from memory: (pos0[b], n_tok[b]) of a chunk -- an invalid
// pair becomes "no work" (bad set) -- or the document starts of the first rows
// of its two query tiles.
struct PfSeq {
    int P, N;
    int lo0, lo1;
    bool bad;
};
template <int kMode>
__device__ __forceinline__ PfSeq pf_seq(const PfGrid &g, int w) {
    PfSeq q;
    q.P = 0;
    q.N = g.T;
    q.lo0 = q.lo1 = 0;
    q.bad = false;
    if constexpr (kMode == kChunkMode) {
        const int b = pf_tiles(w, g).b;
        q.P = g.pos0[b];
        q.N = g.n_tok ? g.n_tok[b] : g.T;
        q.bad = q.P < 0 || q.N < 0 || q.N > g.T || (long long)q.P + q.N > g.Lmax;
        if (q.bad) q.N = 0;
    } else if constexpr (kMode == kDocs) {
        const PfTiles x = pf_tiles(w, g);
        const int32_t *ds = g.doc_start + (size_t)x.b * g.T;
        const int s0 = ds[x.q0];
        const int s1 = x.has1 ? ds[x.q1] : s0;
        q.lo0 = max(0, min(s0, x.q0)) / 128;
        q.lo1 = x.has1 ? max(0, min(s1, x.q1)) / 128 : q.lo0;
    }
    return q;
}
__device__ __forceinline__ PfSeq pf_seq_none() {
    PfSeq q;
    q.P = q.N = q.lo0 = q.lo1 = 0;
    q.bad = false;
    return q;
}

__device__ __forceinline__ PfItem pf_item(int w, const PfGrid &g, PfSeq sq) {
    const PfTiles x = pf_tiles(w, g);
    PfItem it;
    it.b = x.b;
    it.kvh = x.kvh;
    it.h = x.h0;
    it.q0 = x.q0;
    it.h1 = x.h1;
    it.q1 = x.q1;
    it.P = sq.P;
    it.N = sq.N;
    it.lo0 = sq.lo0;
    it.lo1 = sq.lo1;
    const bool has0 = it.q0 < it.N;
    it.has1 = x.has1 && it.q1 < it.N;
    // tile t sees key tiles [lo_t, n_t); tile 1 ends no earlier than tile 0
    it.n0 = has0 ? (it.P + min(it.N, it.q0 + 128) + 127) / 128 : 0;
    it.n1 = it.has1 ? (it.P + min(it.N, it.q1 + 128) + 127) / 128 : 0;
    it.n_kv = it.has1 ? it.n1 : it.n0;
    // keys [0, kv_end) are valid
    const int kv_end = it.P + min(it.N, (it.has1 ? it.q1 : it.q0) + 128);
    it.r_valid = it.n_kv > 0 ? kv_end - 128 * (it.n_kv - 1) : 128;
    if (it.lo1 < it.lo0) it.lo1 = it.lo0;
    return it;
}

// The producer decodes each item once and passes the result through the ring:
// decoding takes a chain of integer divisions, and in the softmax and MMA warps
// that chain sat on the item boundary's critical path (about 0.3 us per item
// at the 8 x 2048 prompt, waiting behind the exponentials for the SFU).
__device__ __forceinline__ void pf_item_put(volatile int *e, int w, const PfItem &I) {
    e[0] = w;
    e[1] = I.b;
    e[2] = I.h;
    e[3] = I.kvh;
    e[4] = I.q0;
    e[5] = I.n0;
    e[6] = I.n1;
    e[7] = I.n_kv;
    e[8] = I.h1;
    e[9] = I.q1;
    e[10] = I.lo0;
    e[11] = I.lo1;
    e[12] = I.P;
    e[13] = I.N;
    e[14] = I.r_valid;
    e[15] = I.has1 ? 1 : 0;
}
// The x-th item of this CTA, decoded, read from the ring (waits for the
// producer); a wait that times out reads as the end.
__device__ __forceinline__ int pf_item_at(PfSync &sy, int x, PfItem &I) {
    if (!ptx::mbar_wait_warp(A(sy.item_full[x & 3]), (x >> 2) & 1)) return -1;
    const volatile int *e = sy.item[x & 3];
    I.b = e[1];
    I.h = e[2];
    I.kvh = e[3];
    I.q0 = e[4];
    I.n0 = e[5];
    I.n1 = e[6];
    I.n_kv = e[7];
    I.h1 = e[8];
    I.q1 = e[9];
    I.lo0 = e[10];
    I.lo1 = e[11];
    I.P = e[12];
    I.N = e[13];
    I.r_valid = e[14];
    I.has1 = e[15] != 0;
    return e[0];
}

template <int D, int kMode>
__device__ void producer(const PfMaps &maps, PfSync &sy, uint8_t *smem, const PfGrid &g,
                         int32_t *status) {
    using S = PfShape<D>;
    int kc = 0, vc = 0, qc = 0;     // K, V tiles and Q pairs this CTA has loaded
    bool ok = true;
    // with fewer than four items per CTA the static dealing pairs long and short
    // items better than first-come order (8 x 1024 MHA prompt: 32.8 against 34.8 us)
    const bool dynamic = g.n_items >= 4 * (int)gridDim.x;
    for (int k = 0; ok; ++k) {
        // take the next item and hand it, with its sequence data, to the other roles
        const int s = k & 3;
        ok = ptx::mbar_wait(A(sy.item_empty[s]), ((k >> 2) & 1) ^ 1);
        if (!ok) break;
        int w = dynamic ? atomicAdd(g.work, 1) : pf_static_w<kMode>(k);
        if (w >= g.n_items) w = -1;
        const PfSeq sq = w >= 0 ? pf_seq<kMode>(g, w) : pf_seq_none();
        const PfItem I = pf_item(w >= 0 ? w : 0, g, sq);
        pf_item_put(sy.item[s], w, I);
        ptx::mbar_arrive(A(sy.item_full[s]));
        if (w < 0) break;
        if (sq.bad) report(status, sq.P < 0 || sq.N < 0 ? GQA_DEV_BAD_LEN : GQA_DEV_CAPACITY);
        if (I.n_kv == 0) continue;
        // The previous item's last S MMA has released the Q tiles.
        ok = ptx::mbar_wait(A(sy.q_empty), (qc & 1) ^ 1);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(A(sy.q_full), S::kTileBytes * (I.has1 ? 2 : 1));
        for (int t = 0; t < (I.has1 ? 2 : 1); ++t)
            for (int kb = 0; kb < S::kBlocks; ++kb)
                ptx::tma_load_4d(ptx::smem_addr(smem + S::kOffQ + t * S::kTileBytes + kb * S::kBlockBytes),
                                 &maps.q, A(sy.q_full), kb * 64, t ? I.h1 : I.h, t ? I.q1 : I.q0, I.b);
        ++qc;
        // K tiles run ahead of V tiles: S(j) needs K(j) one MMA pair before
        // PV(j) needs V(j), and the K ring is the deeper one.
        int jk = I.lo0, jv = I.lo0;
        while (ok && jv < I.n_kv) {
            if (jk < I.n_kv && jk < jv + S::kStagesK) {
                const int st = kc % S::kStagesK;
                ok = ptx::mbar_wait(A(sy.k_empty[st]), ((kc / S::kStagesK) & 1) ^ 1);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(A(sy.k_full[st]), S::kTileBytes);
                for (int kb = 0; kb < S::kBlocks; ++kb)
                    ptx::tma_load_3d(ptx::smem_addr(smem + S::kOffK + st * S::kTileBytes + kb * S::kBlockBytes),
                                     &maps.k, A(sy.k_full[st]), kb * 64, jk * 128, I.b * g.Hkv + I.kvh);
                ++kc;
                ++jk;
            }
            if (jv < jk) {
                const int st = vc % S::kStagesV;
                ok = ptx::mbar_wait(A(sy.v_empty[st]), ((vc / S::kStagesV) & 1) ^ 1);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(A(sy.v_full[st]), S::kTileBytes);
                for (int kb = 0; kb < S::kBlocks; ++kb)
                    ptx::tma_load_3d(ptx::smem_addr(smem + S::kOffV + st * S::kTileBytes + kb * S::kBlockBytes),
                                     &maps.v, A(sy.v_full[st]), kb * 64, jv * 128, I.b * g.Hkv + I.kvh);
                ++vc;
                ++jv;
            }
        }
    }
    if (!ok) {
        report(status, GQA_DEV_TIMEOUT);
        // Let every copy already issued land before the CTA can retire.
        if (qc > 0) ptx::mbar_wait(A(sy.q_full), (qc - 1) & 1);
        for (int j = (kc > S::kStagesK ? kc - S::kStagesK : 0); j < kc; ++j)
            ptx::mbar_wait(A(sy.k_full[j % S::kStagesK]), (j / S::kStagesK) & 1);
        for (int j = (vc > S::kStagesV ? vc - S::kStagesV : 0); j < vc; ++j)
            ptx::mbar_wait(A(sy.v_full[j % S::kStagesV]), (j / S::kStagesV) & 1);
    }
}

template <int D, int kMode>
__device__ void mma_issuer(PfSync &sy, uint8_t *smem, uint32_t tmem, const PfGrid &g,
                           int32_t *status) {
    using S = PfShape<D>;
    const uint32_t go = ptx::elect_one();   // the lane that issues
    constexpr uint32_t idS = ptx::idesc_bf16_f32(128, 128, false);
    constexpr uint32_t idO = ptx::idesc_bf16_f32(128, D, true);
    const uint32_t q_base = ptx::smem_addr(smem + S::kOffQ);
    const uint32_t k_base = ptx::smem_addr(smem + S::kOffK);
    const uint32_t v_base = ptx::smem_addr(smem + S::kOffV);

    auto issue_s = [&](int t, int kst) {
        const uint32_t qa = q_base + t * S::kTileBytes;
        const uint32_t ka = k_base + kst * S::kTileBytes;
#pragma unroll
        for (int ks = 0; ks < S::kKSteps; ++ks) {
            const uint32_t off = (ks >> 2) * S::kBlockBytes + (ks & 3) * 32;
            ptx::mma_ss_if(go, tmem + t * 128, ptx::smem_desc_sw128(qa + off, 16, 1024),
                        ptx::smem_desc_sw128(ka + off, 16, 1024), idS, ks > 0);
        }
        ptx::mma_commit_if(go, A(sy.s_full[t]));
    };
    // O_t (+)= P_t V over key rows [16 k0, 16 k1) of the tile.
    auto issue_pv = [&](int t, int vst, bool acc, int k0, int k1) {
        const uint32_t va = v_base + vst * S::kTileBytes;
#pragma unroll
        for (int ks = k0; ks < k1; ++ks)
            ptx::mma_ts_if(go, tmem + 256 + t * 128, tmem + t * 128 + ks * 8,
                        ptx::smem_desc_sw128(va + ks * 2048, S::kBlockBytes, 1024), idO,
                        (acc || ks > 0) ? 1u : 0u);
    };
    // P_t arrives in two halves (key columns 0-63, then 64-127), and the
    // product with the first half runs while the softmax computes the second
    // (2 % faster on the 8 x 2048 prompt, 4 % on chunks and documents).
    auto issue_pv_halves = [&](int t, int vst, bool acc, int pc) {
        if (!ptx::mbar_wait_warp(A(sy.p_half[t]), pc & 1)) return false;
        ptx::tc_fence_after();
        issue_pv(t, vst, acc, 0, 4);
        if (!ptx::mbar_wait_warp(A(sy.p_full[t]), pc & 1)) return false;
        ptx::tc_fence_after();
        issue_pv(t, vst, true, 4, 8);
        return true;
    };

    int kc = 0, vc = 0, qc = 0;     // K, V tiles and Q pairs consumed
    int pc0 = 0, pc1 = 0;           // P hand-overs received from each softmax group
    bool ok = true;
    for (int k = 0; ok; ++k) {
        PfItem I;
        const int w = pf_item_at(sy, k, I);
        __syncwarp();
        if (w < 0) break;
        if (go) ptx::mbar_arrive(A(sy.item_empty[k & 3]));   // the ring slot has been read
        if (I.n_kv == 0) continue;
        const int kc0 = kc;           // K ring index of key tile lo0
        ok = ptx::mbar_wait_warp(A(sy.q_full), qc & 1) &&
             ptx::mbar_wait_warp(A(sy.k_full[kc0 % S::kStagesK]), (kc0 / S::kStagesK) & 1);
        if (!ok) break;
        ++qc;
        ptx::tc_fence_after();
        // Query tile t covers key tiles [lo_t, n_t): lo_t = 0 except with
        // documents, where tile 1 may start later than tile 0.
        const bool t1_first = I.has1 && I.lo1 == I.lo0;
        issue_s(0, kc0 % S::kStagesK);
        if (t1_first) issue_s(1, kc0 % S::kStagesK);
        ptx::mma_commit_if(go, A(sy.k_empty[kc0 % S::kStagesK]));
        if (I.n_kv - I.lo0 == 1) ptx::mma_commit_if(go, A(sy.q_empty));   // Q no longer read
        for (int j = I.lo0; j < I.n_kv && ok; ++j) {
            const int vst = vc % S::kStagesV;
            ok = ptx::mbar_wait_warp(A(sy.v_full[vst]), (vc / S::kStagesV) & 1);
            if (!ok) break;
            const int jn = j + 1;
            const int kidx = kc0 + (jn - I.lo0);
            const int kst = kidx % S::kStagesK;
            bool k_next = false;
            if (j < I.n0) {
                ok = issue_pv_halves(0, vst, j > I.lo0, pc0);
                if (!ok) break;
                ++pc0;
                if (jn < I.n0) {
                    ok = ptx::mbar_wait_warp(A(sy.k_full[kst]), (kidx / S::kStagesK) & 1);
                    if (!ok) break;
                    k_next = true;
                    issue_s(0, kst);
                } else {
                    ptx::mma_commit_if(go, A(sy.o_final[0]));
                }
            }
            if (I.has1 && j >= I.lo1 && j < I.n1) {
                ok = issue_pv_halves(1, vst, j > I.lo1, pc1);
                if (!ok) break;
                ++pc1;
                if (jn < I.n1) {
                    if (!k_next) {
                        ok = ptx::mbar_wait_warp(A(sy.k_full[kst]), (kidx / S::kStagesK) & 1);
                        if (!ok) break;
                        k_next = true;
                    }
                    issue_s(1, kst);
                } else {
                    ptx::mma_commit_if(go, A(sy.o_final[1]));
                }
            } else if (kMode == kDocs && I.has1 && jn == I.lo1) {
                // tile 1's first scores, on the next key tile
                if (!k_next) {
                    ok = ptx::mbar_wait_warp(A(sy.k_full[kst]), (kidx / S::kStagesK) & 1);
                    if (!ok) break;
                    k_next = true;
                }
                issue_s(1, kst);
            }
            ptx::mma_commit_if(go, A(sy.v_empty[vst]));
            ++vc;
            if (k_next) {
                ptx::mma_commit_if(go, A(sy.k_empty[kst]));
                if (jn == I.n_kv - 1) ptx::mma_commit_if(go, A(sy.q_empty));   // last S of the item
            }
        }
        kc = kc0 + (I.n_kv - I.lo0);
    }
    if (!ok && go) report(status, GQA_DEV_TIMEOUT);
    // No MMA may still be writing tensor memory when it is released.
    ptx::mma_commit_if(go, A(sy.mma_done));
    ptx::mbar_wait_warp(A(sy.mma_done), 0);
}

template <int D, int kMode>
__device__ void softmax_tile(const PfMaps &maps, PfSync &sy, uint8_t *smem, uint32_t tmem, int t,
                             const PfGrid &g, float scale_log2, uint16_t *__restrict__ out,
                             int32_t *status) {
    using S = PfShape<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = t * 128, o_col = 256 + t * 128;
    const int T = g.T;
    int sc = 0, oc = 0;             // scores and outputs of this tile received
    const bool st_issuer = (warp & 3) == 0 && lane == 0;   // issues the group's output stores
    int vc = 0;                     // V tiles of the items before this one
    bool ok = true;
    for (int k = 0; ok; ++k) {
        PfItem I;
        const int w = pf_item_at(sy, k, I);
        __syncwarp();
        if (w < 0) break;
        if (lane == 0) ptx::mbar_arrive(A(sy.item_empty[k & 3]));   // the ring slot has been read
        const int vc0 = vc;
        vc += I.n_kv - I.lo0;
        if (I.n_kv == 0 || (t == 1 && !I.has1)) continue;
        const int q_first = t ? I.q1 : I.q0;
        const int hd = t ? I.h1 : I.h;          // this tile's query head
        const int nt = t == 0 ? I.n0 : I.n1;
        const int jlo = t == 0 ? I.lo0 : I.lo1;
        const int qrow = q_first + row;
        const int lim0 = I.P + q_first;          // the tile's first row sees keys <= lim0
        const int qlim = I.P + qrow;             // this row sees keys <= qlim
        // the group whose last key tile is the item's last one clears that V tile's
        // rows past the last valid key (continuation chunks only)
        const bool clears = kMode == kChunkMode && I.r_valid < 128 && nt == I.n_kv &&
                            (t == 0 ? true : I.n0 < I.n_kv);
        // documents: this row sees keys [dstart, qrow]
        int dstart = 0;
        if constexpr (kMode == kDocs) {
            if (qrow < T) {
                dstart = g.doc_start[(size_t)I.b * T + qrow];
                if (dstart < 0 || dstart > qrow) {
                    report(status, GQA_DEV_BAD_LEN);
                    dstart = qrow;
                }
            }
        }
        float m = -INFINITY, l = 0.f;
        for (int j = jlo; j < nt; ++j) {
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.s_full[t]), sc & 1));
            if (!ok) break;
            ++sc;
            ptx::tc_fence_after();
            uint32_t sv[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::tmem_ld32(lane_addr + s_col + 32 * c, sv[c]);
            ptx::tmem_wait_ld();
#define SV(c) __uint_as_float(sv[(c) >> 5][(c) & 31])
            const int key0 = j * 128;
            if constexpr (kMode == kDocs) {
                if (key0 < dstart || key0 + 127 > qlim) {
                    // this row's valid columns [lo, hi] of the tile, as a bit mask per 32
                    const int lo = dstart - key0, hi = qlim - key0;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int a = lo - 32 * ch, z = hi - 32 * ch;
                        uint32_t msk = 0u;
                        if (z >= 0 && a <= 31)
                            msk = (0xffffffffu >> (31 - min(z, 31))) & (0xffffffffu << max(a, 0));
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (!(msk & (1u << e))) sv[ch][e] = __float_as_uint(-INFINITY);
                    }
                }
            } else if (key0 + 127 > lim0) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (key0 + c > qlim) sv[c >> 5][c & 31] = __float_as_uint(-INFINITY);
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
            if (j > jlo && __any_sync(0xffffffffu, resc)) {
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
            // (with documents a row may see no key yet: m is -inf, its p must be 0)
            const float neg_m = (kMode == kDocs && m == -INFINITY) ? 0.f : -m;
            // The last V tile has landed once its barrier's phase completes; zero
            // its rows past the last valid key, then publish the stores to the
            // tensor core (async proxy) before P is handed over.
            auto clear_v_tail = [&]() {
                if (clears && j == nt - 1) {
                    const int vidx = vc0 + I.n_kv - 1;
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.v_full[vidx % S::kStagesV]),
                                                                 (vidx / S::kStagesV) & 1));
                    if (ok) {
                        uint8_t *vt = smem + S::kOffV + (vidx % S::kStagesV) * S::kTileBytes;
                        const int n16 = (128 - I.r_valid) * 8;   // 16-byte pieces per column block
                        for (int x = row; x < n16 * S::kBlocks; x += 128) {
                            const int kb = x / n16, y = x - kb * n16;
                            *reinterpret_cast<uint4 *>(vt + kb * S::kBlockBytes + I.r_valid * 128 + y * 16) =
                                make_uint4(0, 0, 0, 0);
                        }
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    }
                }
            };
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
                if (c == 1) {
                    clear_v_tail();
                    // first half of P (key columns 0-63) to the tensor core
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(A(sy.p_half[t]));
                }
            }
#undef SV
            l += (la0 + la1) + (lb0 + lb1);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(A(sy.p_full[t]));
        }
        if (ok) ok = __all_sync(0xffffffffu, ptx::mbar_wait(A(sy.o_final[t]), oc & 1));
        if (!ok) break;
        ++oc;
        ptx::tc_fence_after();
        const float inv_l = 1.f / l;
        uint16_t *dst = out + (((size_t)I.b * T + qrow) * g.Hq + hd) * D;
        if (kMode == kPromptLse && qrow < T)   // natural-log LSE of the scaled scores
            g.lse[((size_t)I.b * g.Hq + hd) * g.lse_stride + qrow] =
                (m + log2f(l)) * 0.69314718055994531f;
        if (q_first + 128 <= I.N) {
            // Every row of the tile is an output row: the group writes O into its
            // shared-memory staging (128-byte swizzle, 64 columns at a time) and
            // one thread stores the block with the tensor map, so the global
            // writes are whole lines instead of 16 bytes from 32 rows at once.
            uint8_t *stg = smem + S::kOffO + t * S::kBlockBytes;
#pragma unroll
            for (int cb = 0; cb < S::kBlocks; ++cb) {
                uint32_t o[64];
                ptx::tmem_ld32(lane_addr + o_col + 64 * cb, *reinterpret_cast<uint32_t(*)[32]>(o));
                if (64 * cb + 32 < D)
                    ptx::tmem_ld32(lane_addr + o_col + 64 * cb + 32,
                                   *reinterpret_cast<uint32_t(*)[32]>(o + 32));
                ptx::tmem_wait_ld();
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    w[e] = 64 * cb + 2 * e < D
                               ? pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                             __uint_as_float(o[2 * e + 1]) * inv_l)
                               : 0u;
                if (st_issuer) ptx::bulk_wait_read0();     // the last store has read the staging
                ptx::named_bar_sync(1 + t, 128);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(stg + row * 128 + ((c ^ (row & 7)) << 4)) =
                        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                ptx::fence_proxy_async_shared();
                ptx::named_bar_sync(1 + t, 128);
                if (st_issuer) {
                    ptx::tma_store_4d(&maps.o, ptx::smem_addr(stg), 64 * cb, hd, q_first, I.b);
                    ptx::bulk_commit();
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(lane_addr + o_col + 32 * c, o);
                ptx::tmem_wait_ld();
                uint32_t w4[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w4[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                        __uint_as_float(o[2 * e + 1]) * inv_l);
                if (qrow < I.N) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + 32 * c);
                    d4[0] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    d4[1] = make_uint4(w4[4], w4[5], w4[6], w4[7]);
                    d4[2] = make_uint4(w4[8], w4[9], w4[10], w4[11]);
                    d4[3] = make_uint4(w4[12], w4[13], w4[14], w4[15]);
                }
            }
        }
        // the next item's first P hand-over (after this read of O) lets the
        // MMA overwrite O with that item's first product
        ptx::tc_fence_before();
    }
    if (st_issuer) ptx::bulk_wait0();          // the output stores have completed
    if (!ok && lane == 0) report(status, GQA_DEV_TIMEOUT);
}

template <int D, int kMode>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const __grid_constant__ PfMaps maps, uint16_t *__restrict__ out, int B, int T,
               int Hq, int Hkv, int Lmax, const int32_t *__restrict__ pos0,
               const int32_t *__restrict__ n_tok, const int32_t *__restrict__ doc_start,
               float *__restrict__ lse, float scale_log2, int n_pairs, int slot,
               int32_t *status) {
    using S = PfShape<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ PfSync sy;
    PfGrid g;
    g.n_pairs = n_pairs;
    g.B = B;
    g.T = T;
    g.Hq = Hq;
    g.Hkv = Hkv;
    g.Lmax = Lmax;
    g.pos0 = pos0;
    g.n_tok = n_tok;
    g.doc_start = doc_start;
    g.lse = lse;
    g.lse_stride = (T + 3) & ~3;
    g.n_items = n_pairs * Hkv * B;
    g.work = &g_pf_work[slot];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) {
            ptx::mbar_init(A(sy.item_full[i]), 1);
            ptx::mbar_init(A(sy.item_empty[i]), kItemReaders);
        }
        ptx::mbar_init(A(sy.q_full), 1);
        ptx::mbar_init(A(sy.q_empty), 1);
        for (int i = 0; i < S::kStagesK; ++i) {
            ptx::mbar_init(A(sy.k_full[i]), 1);
            ptx::mbar_init(A(sy.k_empty[i]), 1);
        }
        for (int i = 0; i < S::kStagesV; ++i) {
            ptx::mbar_init(A(sy.v_full[i]), 1);
            ptx::mbar_init(A(sy.v_empty[i]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(A(sy.s_full[t]), 1);
            ptx::mbar_init(A(sy.p_half[t]), 4);   // one elected lane per softmax warp
            ptx::mbar_init(A(sy.p_full[t]), 4);
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
    // The kernel is a programmatic dependent of the preceding one (normally the
    // append that rotated q and filled the cache, or the kernel that computed
    // pos0, n_tok or doc_start): every role reads what that kernel wrote -- the
    // producer its tiles, all roles the per-sequence positions, counts and
    // document starts -- so every thread waits for it once the prologue above
    // (barriers, tensor memory, descriptor prefetch) is done.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp >= 8) {
        ptx::regs_dec<kControlRegs>();
        if (warp == kTmaWarp) {
            if (lane == 0) producer<D, kMode>(maps, sy, smem, g, status);
            __syncwarp();
        } else if (warp == kMmaWarp) {
            mma_issuer<D, kMode>(sy, smem, tmem, g, status);   // the whole warp
            __syncwarp();
        }
    } else {
        ptx::regs_inc<kSoftmaxRegs>();
        softmax_tile<D, kMode>(maps, sy, smem, tmem, warp >> 2, g, scale_log2, out, status);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && g.n_items >= 4 * (int)gridDim.x) {   // dynamic dealing: the last
        __threadfence();                                             // CTA out resets the counter
        if (atomicAdd(&g_pf_done[slot], 1u) == gridDim.x - 1) {
            g_pf_work[slot] = 0;
            g_pf_done[slot] = 0;
            __threadfence();
        }
    }
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
template <int D>
gqa_status launch_prefill(const void *q, const void *kc, const void *vc, void *out, int B, int T,
                          int Hq, int Hkv, int Lmax, const int32_t *pos0, const int32_t *n_tok,
                          const int32_t *doc_start, float *lse, float scale_log2,
                          int32_t *status, cudaStream_t s) {
    using S = PfShape<D>;
    PfMaps maps;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T, (cuuint64_t)B};
        const cuuint64_t str[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2,
                                   (cuuint64_t)T * Hq * D * 2};
        const cuuint32_t box[4] = {64, 1, 128, 1};
        if (!encode(&maps.q, q, 4, dims, str, box)) return GQA_ERR_CUDA;
        if (!encode(&maps.o, out, 4, dims, str, box)) return GQA_ERR_CUDA;
    }
    {
        // A prompt (no pos0): rows beyond T are outside the map, so the copies
        // zero-fill them and the unused cache slots (whatever they hold) are
        // never read.  A continuation chunk reads up to slot pos0 + n_tok - 1,
        // so its maps span the whole cache.
        const cuuint64_t rows = pos0 ? (cuuint64_t)Lmax : (cuuint64_t)T;
        const cuuint64_t dims[3] = {(cuuint64_t)D, rows, (cuuint64_t)B * Hkv};
        const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)Lmax * D * 2};
        const cuuint32_t box[3] = {64, 128, 1};
        if (!encode(&maps.k, kc, 3, dims, str, box)) return GQA_ERR_CUDA;
        if (!encode(&maps.v, vc, 3, dims, str, box)) return GQA_ERR_CUDA;
    }
    auto kern = pos0 ? prefill_kernel<D, kChunkMode>
                     : doc_start ? prefill_kernel<D, kDocs>
                     : lse ? prefill_kernel<D, kPromptLse> : prefill_kernel<D, kPrompt>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem) !=
        cudaSuccess)
        return GQA_ERR_CUDA;
    // The warpgroup register split assumes the launch allocation of kLaunchRegs per
    // thread; with any other count the increases could not be satisfied, so refuse.
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return GQA_ERR_CUDA;
    if (attr.numRegs != kLaunchRegs) return GQA_ERR_UNSUPPORTED;
    // items per (b, KV head): its (query tile, head) tiles two at a time
    const int n_pairs = (((T + 127) / 128) * (Hq / Hkv) + 1) / 2;
    const long long items = (long long)n_pairs * Hkv * B;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GQA_ERR_CUDA;
    const long long grid = items < sms ? items : sms;   // persistent: one CTA per SM
    // Programmatic dependent launch: the prologue (barriers, tensor memory,
    // descriptor prefetch) overlaps the tail of the preceding kernel; every
    // thread then waits for that kernel before it reads anything.
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
    static std::atomic<unsigned> next_slot{0};
    const int slot = (int)(next_slot.fetch_add(1, std::memory_order_relaxed) % kWorkSlots);
    if (cudaLaunchKernelEx(&cfg, kern, maps, static_cast<uint16_t *>(out), B, T, Hq, Hkv, Lmax,
                           pos0, n_tok, doc_start, lse, scale_log2, n_pairs, slot,
                           status) != cudaSuccess)
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

namespace {

gqa_status prefill_entry(const void *q, const void *k_cache, const void *v_cache, void *out,
                         const int32_t *pos0, const int32_t *n_tok, const int32_t *doc_start,
                         float *lse, int max_pos0_host, int B, int T, int Hq, int Hkv, int D,
                         int Lmax, float scale, int32_t *status_dev, void *stream) {
    using namespace gqa_host;
    if (!q || !k_cache || !v_cache || !out || B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Lmax < 1)
        return GQA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return GQA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(pos0) & 3u) || (reinterpret_cast<uintptr_t>(n_tok) & 3u) ||
        (reinterpret_cast<uintptr_t>(doc_start) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return GQA_ERR_INVALID_ARG;
    if (!head_dim_ok(D)) return GQA_ERR_UNSUPPORTED;
    if (Lmax % 128 != 0) return GQA_ERR_INVALID_ARG;
    if (max_pos0_host < 0) return GQA_ERR_INVALID_ARG;
    if ((long long)max_pos0_host + T > Lmax) return GQA_ERR_CAPACITY;
    // work items: the (query tile, head) tiles of each (b, KV head), two at a time
    if (((long long)((T + 127) / 128) * (Hq / Hkv) + 1) / 2 * Hkv * B > 0x7fffffffLL)
        return GQA_ERR_INVALID_ARG;
    if (!gqa::device_is_sm100()) return GQA_ERR_UNSUPPORTED;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
    const float sl2 = sc * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (D) {
        case 64: return gqa::launch_prefill<64>(q, k_cache, v_cache, out, B, T, Hq, Hkv, Lmax, pos0, n_tok, doc_start, lse, sl2, status_dev, s);
        case 96: return gqa::launch_prefill<96>(q, k_cache, v_cache, out, B, T, Hq, Hkv, Lmax, pos0, n_tok, doc_start, lse, sl2, status_dev, s);
        default: return gqa::launch_prefill<128>(q, k_cache, v_cache, out, B, T, Hq, Hkv, Lmax, pos0, n_tok, doc_start, lse, sl2, status_dev, s);
    }
}

}  // namespace

extern "C" gqa_status gqa_prefill(const void *q, const void *k_cache, const void *v_cache,
                                  void *out, int B, int T, int Hq, int Hkv, int D, int Lmax,
                                  float scale, int32_t *status_dev, void *stream) {
    return prefill_entry(q, k_cache, v_cache, out, nullptr, nullptr, nullptr, nullptr, 0, B, T, Hq,
                         Hkv, D, Lmax, scale, status_dev, stream);
}

extern "C" gqa_status gqa_prefill_lse(const void *q, const void *k_cache, const void *v_cache,
                                      void *out, float *lse, int B, int T, int Hq, int Hkv, int D,
                                      int Lmax, float scale, int32_t *status_dev, void *stream) {
    if (!lse) return GQA_ERR_INVALID_ARG;
    return prefill_entry(q, k_cache, v_cache, out, nullptr, nullptr, nullptr, lse, 0, B, T, Hq,
                         Hkv, D, Lmax, scale, status_dev, stream);
}

extern "C" gqa_status gqa_prefill_chunk(const void *q, const void *k_cache, const void *v_cache,
                                        void *out, const int32_t *pos0, const int32_t *n_tok,
                                        int max_pos0_host, int B, int T, int Hq, int Hkv, int D,
                                        int Lmax, float scale, int32_t *status_dev, void *stream) {
    if (!pos0) return GQA_ERR_INVALID_ARG;
    return prefill_entry(q, k_cache, v_cache, out, pos0, n_tok, nullptr, nullptr, max_pos0_host, B,
                         T, Hq, Hkv, D, Lmax, scale, status_dev, stream);
}

extern "C" gqa_status gqa_prefill_docs(const void *q, const void *k_cache, const void *v_cache,
                                       void *out, const int32_t *doc_start, int B, int T, int Hq,
                                       int Hkv, int D, int Lmax, float scale, int32_t *status_dev,
                                       void *stream) {
    if (!doc_start) return GQA_ERR_INVALID_ARG;
    return prefill_entry(q, k_cache, v_cache, out, nullptr, nullptr, doc_start, nullptr, 0, B, T,
                         Hq, Hkv, D, Lmax, scale, status_dev, stream);
}

// ---------------------------------------------------------------------------
// gqa_doc_start: per-token document ids -> first position of each document
// ---------------------------------------------------------------------------
namespace {

// One thread per token: the first index t' <= t whose id equals id[t], by binary
// search (ids are non-decreasing along a sequence; a decrease is reported).  It
// lets a programmatic dependent (the documents prefill) start its prologue at
// once; that kernel waits for this one to complete before reading doc_start.
__global__ void __launch_bounds__(256)
doc_start_kernel(const int32_t *__restrict__ doc_id, int32_t *__restrict__ doc_start, int B,
                 int T, int32_t *status) {
    asm volatile("griddepcontrol.launch_dependents;");
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)B * T) return;
    const int b = (int)(i / T), t = (int)(i - (long long)b * T);
    const int32_t *id = doc_id + (size_t)b * T;
    const int32_t me = id[t];
    if (t > 0 && id[t - 1] > me) gqa::report(status, GQA_DEV_BAD_LEN);
    int lo = 0, hi = t;                    // first index in [0, t] with id >= me
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (id[mid] >= me) hi = mid;
        else lo = mid + 1;
    }
    doc_start[i] = lo;
}

}  // namespace

extern "C" gqa_status gqa_doc_start(const int32_t *doc_id, int32_t *doc_start, int B, int T,
                                    int32_t *status_dev, void *stream) {
    if (!doc_id || !doc_start || B < 1 || T < 1) return GQA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(doc_id) & 3u) || (reinterpret_cast<uintptr_t>(doc_start) & 3u))
        return GQA_ERR_INVALID_ARG;
    const long long n = (long long)B * T;
    if (n > 0x7fffffffLL * 256LL) return GQA_ERR_INVALID_ARG;
    doc_start_kernel<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        doc_id, doc_start, B, T, status_dev);
    return gqa_host::launch_status();
}
