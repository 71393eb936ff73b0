// Paged prefill / chunked-prefill attention on 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory).
//
// What is computed: the prefill phase ("大模型推理加速与显存黑科技 (Inference
// Acceleration & KV Cache)" §1: the whole prompt is processed in parallel)
// over the paged cache ("LLM 推理优化：KV Cache、PagedAttention 与量化" §2.2):
// a chunk of q_len new tokens per sequence, already appended to the cache, each
// attending causally to every earlier token and to itself:
//   out[s][j][h] = softmax(scale * q[s][j][h] . K_t) V_t,  t = 0 .. L_s - q_len + j,
// with the Attention(Q,K,V) formula of the same page's §2 and the tiled
// online softmax of its §4.2.  Query head h reads KV head h / (Hq/Hkv).
//
// Design (sm_100a): one CTA per SM-sized work item (sequence, kv head, two
// consecutive tiles of 128 query rows); the rows of a tile are (position,
// head-in-group) pairs, so both tiles share every K/V tile staged for their KV
// head.  Per 128-token stage and tile t:
//   S_t = Q_t K^T  tcgen05.mma kind::f16, M128 N128 K128, fp32 in tensor memory
//   softmax        4 warps per tile, thread i owns row i (= TMEM lane i): no
//                  shuffles; two passes over the 128 scores (max, then exp2)
//   O_t += P_t V   tcgen05.mma, M128 N128 K128, P fp16 in tensor memory (it is
//                  written over S_t), V from shared memory
// Warp roles: warps 0-7 softmax / epilogue (4 per tile), warp 8 TMA producer,
// warp 9 TMEM allocation + MMA issue.  Tensor memory: S_t and O_t for both
// tiles (512 columns).  S is single-buffered per tile (S_t(j+1) waits for
// P V_t(j)); the two tiles ping-pong: while one tile is in its softmax the
// other's MMAs run.  The softmax does its fp32 arithmetic two values per
// instruction (packed f32x2 multiply-add and add, three-input maximum).
// K and V arrive through separate two-slot rings
// (32 KB slots) shared by the tiles; the producer polls both rings and fills
// whichever slot frees first.  The MMA warp issues in the one order in which
// the tiles' work becomes ready (S_0 and S_1 of the first stage, then per
// stage P V_0, the next S_0, P V_1, the next S_1), blocking on each barrier so
// that it wakes as soon as the barrier completes.  O is rescaled lazily: only
// when a row's running maximum grows by more than 2^8 (weights stay below 2^8
// otherwise, well within fp16 and fp32).  Every wait is bounded; tensor memory
// is released on every path out of the kernel.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "../../include/paged_kv.h"
#include "kv_device.h"
#include "kv_ptx.cuh"
#include "kv_status.h"

namespace pkv_prefill {

using namespace pkv;

constexpr int D = 128;          // head dim served by this kernel
constexpr int M = 128;          // query rows per tile (TMEM lanes)
constexpr int NT = 2;           // query tiles per CTA; they share every K/V stage
constexpr int TS = 128;         // tokens per stage (S columns)
constexpr int KV_SLOTS = 2;     // slots in each of the K and V rings
constexpr int SM_WARPS = 4 * NT;               // softmax warps: 4 per tile
constexpr int PRODUCER_WARP = SM_WARPS;
constexpr int MMA_WARP = SM_WARPS + 1;
constexpr int NTHREADS = 32 * (SM_WARPS + 2);
// tensor memory: tile t's S at t*TS (P is written over its first TS/2
// columns), its O at O_COL + t*D: 2 * (128 + 128) = 512 columns
constexpr int O_COL = NT * TS;
constexpr int TMEM_COLS = O_COL + NT * D;
static_assert(TMEM_COLS == 512, "tensor memory layout");
constexpr uint64_t kWait = 2000000000ull;
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kRescaleThreshold = 8.f;  // log2 units

// shared memory layout (bytes, from a 1024-aligned base)
constexpr int Q_OFF = 0;                        // tile t: [2 halves][128 rows][128 B]
constexpr int Q_TILE = 2 * M * 128;             // 32 KB
constexpr int Q_BYTES = NT * Q_TILE;
constexpr int KV_HALF = TS * 128;               // 16 KB: one 64-column half of a stage
constexpr int SLOT_BYTES = 2 * KV_HALF;         // 32 KB: K (or V) of one stage
constexpr int K_OFF = Q_OFF + Q_BYTES;          // K ring
constexpr int V_OFF = K_OFF + KV_SLOTS * SLOT_BYTES;  // V ring
constexpr int BAR_OFF = V_OFF + KV_SLOTS * SLOT_BYTES;
// barriers: q_full, kfull[KS], kempty[KS], vfull[KS], vempty[KS], per tile
// s_full, s_free, p_full; drain
constexpr int NBARS = 1 + 4 * KV_SLOTS + 3 * NT + 1;
constexpr int TMEM_SLOT_OFF = BAR_OFF + NBARS * 8;
constexpr int SMEM_USED = TMEM_SLOT_OFF + 16;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;
static_assert(SMEM_ALLOC <= 232448, "one CTA per SM must fit");

// Progress watchdog for the producer's polling loop: true once `limit` ns of
// wall time have passed without progress (the clock is read every 1024 idle
// polls); a limit below kFineWaitNs expires at the first idle poll.
struct Idle {
    uint32_t n = 0;
    uint64_t t0 = 0;
    __device__ __forceinline__ void reset() { n = 0; }
    __device__ __forceinline__ bool expired(uint64_t limit)
    {
        if (limit < kFineWaitNs) return true;
        if ((++n & 1023u) != 0) return false;
        const uint64_t now = globaltimer_ns();
        if (n == 1024u) {
            t0 = now;
            return false;
        }
        return now - t0 > limit;
    }
};

struct Params {
    const __half* q;
    __half* out;
    const int32_t* block_tables;
    const int32_t* context_lens;
    int* err;
    int32_t max_blocks, B, q_len, Hq, Hkv, G, bs, num_blocks, tiles_per_head;
    float scale_log2;
    uint64_t idle_ns;  // the loader's limit without progress
};

// ---- packed fp32 arithmetic of the softmax (two lanes of work per instruction)
__device__ __forceinline__ uint64_t f32x2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_split(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// maximum of three in one instruction
__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmQ, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int abort_flag;
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = sb + BAR_OFF;
    const uint32_t q_full = bar0;
    // K and V rings are separate and shared by the NT query tiles: a K slot
    // is free once every tile's S = Q K^T of its stage is done, a V slot once
    // every tile's P V is.
    auto kfull = [&](int i) { return bar0 + 8 * (1 + i); };
    auto kempty = [&](int i) { return bar0 + 8 * (1 + KV_SLOTS + i); };
    auto vfull = [&](int i) { return bar0 + 8 * (1 + 2 * KV_SLOTS + i); };
    auto vempty = [&](int i) { return bar0 + 8 * (1 + 3 * KV_SLOTS + i); };
    // per tile t: S full, S free (the P V that read P over it is done), P
    // written.  S is single-buffered per tile: S_t(j+1) waits for P V_t(j),
    // which needs all four warps' arrive for stage j, so a warp never passes
    // stage j before the others of its tile arrived for it.
    auto s_full = [&](int t) { return bar0 + 8 * (1 + 4 * KV_SLOTS + 3 * t); };
    auto s_free = [&](int t) { return bar0 + 8 * (2 + 4 * KV_SLOTS + 3 * t); };
    auto p_full = [&](int t) { return bar0 + 8 * (3 + 4 * KV_SLOTS + 3 * t); };
    const uint32_t drain = bar0 + 8 * (1 + 4 * KV_SLOTS + 3 * NT);

    // work item: NT consecutive tiles of one (sequence, kv head)
    const int pair = blockIdx.x % p.tiles_per_head;
    const int kvh = (blockIdx.x / p.tiles_per_head) % p.Hkv;
    const int s = blockIdx.x / (p.tiles_per_head * p.Hkv);
    const int pos_per_tile = M / p.G;
    const int jbase = pair * NT * pos_per_tile;            // first window position
    int jn_all = p.q_len - jbase;
    if (jn_all > NT * pos_per_tile) jn_all = NT * pos_per_tile;  // positions in this CTA
    int32_t L = __ldg(p.context_lens + s);
    if (L > p.max_blocks * p.bs) {
        if (threadIdx.x == 0) atomicOr(p.err, KV_DEV_BAD_BLOCK);
        L = p.max_blocks * p.bs;
    }
    // last token any row of this CTA may see (exclusive end)
    int kv_end = L - p.q_len + jbase + jn_all;
    if (kv_end > L) kv_end = L;
    if (kv_end < 0) kv_end = 0;
    const int nst = (kv_end + TS - 1) / TS;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(q_full, 1);
        for (int i = 0; i < KV_SLOTS; ++i) {
            mbar_init(kfull(i), 1);
            mbar_init(kempty(i), 1);
            mbar_init(vfull(i), 1);
            mbar_init(vempty(i), 1);
        }
        for (int t = 0; t < NT; ++t) {
            mbar_init(s_full(t), 1);
            mbar_init(s_free(t), 1);
            mbar_init(p_full(t), 4);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(sb + TMEM_SLOT_OFF, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + TMEM_SLOT_OFF);

    if (warp == PRODUCER_WARP) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = l2_policy_evict_first();
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmQ);
            // Q tile t: rows r = (j - j0_t) * G + g; one box per 64-column half,
            // G heads x pos_per_tile positions (positions past the chunk are
            // never stored: their rows see no key)
            mbar_arrive_expect_tx(q_full, Q_BYTES);
            for (int t = 0; t < NT; ++t) {
                const int z = s * p.q_len + jbase + t * pos_per_tile;
                for (int h = 0; h < 2; ++h)
                    asm volatile(
                        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(sb + Q_OFF + t * Q_TILE + h * M * 128),
                        "l"(reinterpret_cast<uint64_t>(&tmQ)), "r"(h * 64), "r"(kvh * p.G), "r"(z),
                        "r"(q_full)
                        : "memory");
            }
        }
        // K (or V) of stage j into its (free) ring slot: block `lane` of the
        // stage -> rows [lane*bs, lane*bs+bs) of each 64-column half of the slot.
        auto issue = [&](int j, bool is_v) {
            const int slot = j % KV_SLOTS;
            const uint32_t fullb = is_v ? vfull(slot) : kfull(slot);
            const int t0 = j * TS;
            int ntok = kv_end - t0;
            if (ntok > TS) ntok = TS;
            const int nblk = (ntok + p.bs - 1) / p.bs;
            int32_t id = -1;
            if (lane < nblk) id = __ldg(p.block_tables + (int64_t)s * p.max_blocks + t0 / p.bs + lane);
            const bool bad = lane < nblk && (id < 0 || id >= p.num_blocks);
            const bool load = lane < nblk && !bad;
            const unsigned lmask = __ballot_sync(0xffffffffu, load);
            if (!is_v && __any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err, KV_DEV_BAD_BLOCK);
            if (lane == 0)
                mbar_arrive_expect_tx(fullb, (uint32_t)__popc(lmask) * (uint32_t)(p.bs * D * 2));
            __syncwarp();
            if (load) {
                const uint32_t dst = sb + (is_v ? V_OFF : K_OFF) + slot * SLOT_BYTES +
                                     (uint32_t)(lane * p.bs * 128);
                const int32_t y = (id * p.Hkv + kvh) * p.bs;
                const CUtensorMap* tm = is_v ? &tmV : &tmK;
                tma_load_2d(dst, tm, 0, y, fullb, pol);
                tma_load_2d(dst + KV_HALF, tm, 64, y, fullb, pol);
            }
        };
        // slot of stage j free?  (its previous use, stage j - KV_SLOTS, consumed
        // by every tile; lane 0 decides for the warp)
        auto slot_free = [&](int j, bool is_v) {
            bool f = true;
            if (j >= KV_SLOTS)
                f = mbar_test(is_v ? vempty(j % KV_SLOTS) : kempty(j % KV_SLOTS), ((j / KV_SLOTS) - 1) & 1);
            return __shfl_sync(0xffffffffu, f ? 1 : 0, 0) != 0;
        };
        // Poll both rings and issue whichever slot frees first.
        bool ok = true;
        int k_issued = 0, v_issued = 0;
        Idle idle;
        while (k_issued < nst || v_issued < nst) {
            bool prog = false;
            if (k_issued < nst && slot_free(k_issued, false)) {
                issue(k_issued++, false);
                prog = true;
            }
            if (v_issued < k_issued && slot_free(v_issued, true)) {
                issue(v_issued++, true);
                prog = true;
            }
            if (prog) {
                idle.reset();
                continue;
            }
            if (__shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&abort_flag), 0) ||
                __shfl_sync(0xffffffffu, idle.expired(p.idle_ns) ? 1 : 0, 0)) {
                ok = false;
                break;
            }
        }
        if (!ok && lane == 0) {
            atomicOr(p.err, KV_DEV_TIMEOUT);
            abort_flag = 1;
        }
        // drain: the last copy into each slot of each ring must have landed
        for (int i = lane; i < KV_SLOTS; i += 32) {
            if (i < k_issued) {
                const int n_i = (k_issued - i + KV_SLOTS - 1) / KV_SLOTS;
                if (!mbar_wait_bounded(kfull(i), (n_i - 1) & 1, kWait)) atomicOr(p.err, KV_DEV_TIMEOUT);
            }
            if (i < v_issued) {
                const int n_i = (v_issued - i + KV_SLOTS - 1) / KV_SLOTS;
                if (!mbar_wait_bounded(vfull(i), (n_i - 1) & 1, kWait)) atomicOr(p.err, KV_DEV_TIMEOUT);
            }
        }
        if (lane == 0 && !mbar_wait_bounded(q_full, 0, kWait)) atomicOr(p.err, KV_DEV_TIMEOUT);
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t idS = idesc_f16(M, TS, false);
            const uint32_t idO = idesc_f16(M, D, true);
            bool ok = mbar_wait_bounded(q_full, 0, kWait);
            tc_fence_after();
            // S_t(j): S = Q_t K^T, M128 N128, 8 k-steps of 16 dims (4 per
            // 64-dim half); the last tile's issue releases the shared K slot.
            auto issue_S = [&](int t, int j) {
                tc_fence_after();
                const uint32_t qa = sb + Q_OFF + t * Q_TILE;
                const uint32_t kb = sb + K_OFF + (j % KV_SLOTS) * SLOT_BYTES;
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k & 3) * 32;
                    const uint64_t a = smem_desc(qa + (k >> 2) * M * 128 + off, 16, 1024);
                    const uint64_t bd = smem_desc(kb + (k >> 2) * KV_HALF + off, 16, 1024);
                    umma_f16(tmem + t * TS, a, bd, idS, k > 0 ? 1u : 0u);
                }
                umma_commit(s_full(t));
                if (t == NT - 1) umma_commit(kempty(j % KV_SLOTS));  // K of stage j consumed
            };
            // P V_t(j): O_t += P V over 8 k-steps of 16 tokens.  P: fp16 pairs in
            // the first 64 columns of S_t.  V is MN-major (dims contiguous):
            // 64-dim groups KV_HALF apart, 8-token groups 1 KB apart.  Its
            // completion frees S_t for the tile's next S.
            auto issue_PV = [&](int t, int j) {
                tc_fence_after();
                const uint32_t vb = sb + V_OFF + (j % KV_SLOTS) * SLOT_BYTES;
                for (int k = 0; k < 8; ++k) {
                    const uint64_t bd = smem_desc(vb + k * 16 * 128, KV_HALF, 1024);
                    umma_f16_ts(tmem + O_COL + t * D, tmem + t * TS + k * 8, bd, idO,
                                (j > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(s_free(t));
                if (t == NT - 1) umma_commit(vempty(j % KV_SLOTS));  // V of stage j consumed
            };
            // Issue order: S_0(0), S_1(0), then per stage j: P V_0(j),
            // S_0(j+1), P V_1(j), S_1(j+1) (tile 0's softmax of a stage
            // usually finishes first: its S was issued first).  Blocking waits
            // wake on each barrier as it completes; while one tile is in its
            // softmax, the other's MMAs keep the tensor pipe busy.
            if (ok && nst > 0) ok = mbar_wait_bounded(kfull(0), 0, kWait);
            if (ok && nst > 0) {
                for (int t = 0; t < NT; ++t) issue_S(t, 0);
            }
            for (int j = 0; j < nst && ok; ++j) {
                for (int t = 0; t < NT && ok; ++t) {
                    ok = mbar_wait_bounded(p_full(t), j & 1, kWait) &&
                         mbar_wait_bounded(vfull(j % KV_SLOTS), (j / KV_SLOTS) & 1, kWait);
                    if (!ok) break;
                    issue_PV(t, j);
                    if (j + 1 < nst) {
                        ok = mbar_wait_bounded(kfull((j + 1) % KV_SLOTS), ((j + 1) / KV_SLOTS) & 1, kWait) &&
                             mbar_wait_bounded(s_free(t), j & 1, kWait);
                        if (!ok) break;
                        issue_S(t, j + 1);
                    }
                }
            }
            if (!ok) {
                atomicOr(p.err, KV_DEV_TIMEOUT);
                abort_flag = 1;
            }
            // everything issued must have finished before tensor memory is freed
            umma_commit(drain);
            if (!mbar_wait_bounded(drain, 0, kWait)) atomicOr(p.err, KV_DEV_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        // warps 4t .. 4t+3 serve tile t; thread row r = TMEM lane r
        const int t = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_col = (uint32_t)(t * TS), o_col = (uint32_t)(O_COL + t * D);
        const int jr = t * pos_per_tile + r / p.G;    // position within this CTA's window
        const bool row_ok = jr < jn_all;
        const int lim = L - p.q_len + jbase + jr;     // last visible token (inclusive)
        const float sl2 = p.scale_log2;
        float m = kNegInf, l = 0.f;
        bool ok = true;
        // 64 scores of half h of the stage, masked past what the row sees
        auto load_half = [&](int h, int vis, bool full, float (&sv)[64]) {
            float t32[32];
            tmem_ld32(lane_base + s_col + 64 * h, t32);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[i] = t32[i];
            tmem_ld32(lane_base + s_col + 64 * h + 32, t32);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[32 + i] = t32[i];
            tmem_wait_ld();
            if (!full) {
#pragma unroll
                for (int c = 0; c < 64; ++c) sv[c] = 64 * h + c < vis ? sv[c] : kNegInf;
            }
        };
        for (int j = 0; j < nst && ok; ++j) {
            const int slot = j % KV_SLOTS;
            ok = mbar_wait_bounded(s_full(t), j & 1, kWait);
            if (!ok) break;
            tc_fence_after();
            const int t0 = j * TS;
            int ntok = kv_end - t0;                   // staged tokens (< TS: last stage)
            if (ntok > TS) ntok = TS;
            int vis = lim - t0 + 1;                   // columns this row may see
            if (vis > ntok) vis = ntok;
            if (!row_ok) vis = 0;
            const bool full = __all_sync(0xffffffffu, vis >= TS);
            // pass 1: the row maximum (raw scores; scale > 0 commutes with it)
            float mx4[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
            for (int h = 0; h < 2; ++h) {
                float sv[64];
                load_half(h, vis, full, sv);
#pragma unroll
                for (int c = 0; c < 64; c += 8)
#pragma unroll
                    for (int k = 0; k < 4; ++k) mx4[k] = max3(mx4[k], sv[c + 2 * k], sv[c + 2 * k + 1]);
            }
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
            // S_t(j) was issued after P V_t(j-1) finished and P V_t(j) waits for
            // this warp's arrive: O is quiet, a rescale needs no wait.
            const bool grow = mx > m + kRescaleThreshold;
            if (__any_sync(0xffffffffu, grow)) {
                const float mn = grow ? mx : m;
                const float alpha = mn == kNegInf ? 1.f : ex2(m - mn);
                if (j >= 1) {
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        float o32[32];
                        tmem_ld32(lane_base + o_col + c0, o32);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o32[i] *= alpha;
                        tmem_st32(lane_base + o_col + c0, o32);
                    }
                    tmem_wait_st();
                }
                l *= alpha;
                m = mn;
            }
            const float mu = m == kNegInf ? 0.f : m;
            // pass 2: fp16 weights packed in pairs into the first 64 columns of
            // S_t (half h -> columns 32h ..; those S columns are already read);
            // the exponents scale*s - mu and the row sum two at a time
            uint64_t ps2[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
            const uint64_t sl2x2 = f32x2(sl2, sl2), nmu2 = f32x2(-mu, -mu);
            for (int h = 0; h < 2; ++h) {
                float sv[64];
                load_half(h, vis, full, sv);
                float pw[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float x0, x1;
                    f32x2_split(fma_f32x2(f32x2(sv[2 * e], sv[2 * e + 1]), sl2x2, nmu2), x0, x1);
                    const float a = ex2(x0), bq = ex2(x1);
                    ps2[e & 1] = add_f32x2(ps2[e & 1], f32x2(a, bq));
                    pw[e] = __uint_as_float(pack_half2(a, bq));
                }
                tmem_st32(lane_base + s_col + 32 * h, pw);
            }
            {
                float a0, a1, b0, b1;
                f32x2_split(ps2[0], a0, a1);
                f32x2_split(ps2[1], b0, b1);
                l += (a0 + b0) + (a1 + b1);
            }
            // V rows past the staged tokens must be finite zeros for the MMA
            // (tile 0 writes them; tile 1's P V is issued after tile 0's, which
            // waited for these writes).  The copy of this stage's V must have
            // landed first; V of stage j+KS cannot start before P V of stage j,
            // so the phase is this one.
            if (t == 0 && ntok < TS) {
                ok = mbar_wait_bounded(vfull(slot), (j / KV_SLOTS) & 1, kWait);
                if (!ok) break;
                uint8_t* vb = smem + V_OFF + slot * SLOT_BYTES;
                for (int i = r; i < (TS - ntok) * 16; i += M) {
                    const int row = ntok + i / 16, ch = i % 16;  // 16 chunks: 2 halves x 8
                    *reinterpret_cast<uint4*>(vb + (ch >> 3) * KV_HALF + row * 128 + ((ch & 7) << 4)) =
                        make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async();  // the V zeros above are read by the tensor core
            tmem_wait_st();
            tc_fence_before();
            // the tile's 128 softmax threads wrote their part: one arrive per warp
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(t));
        }
        // epilogue: O / l, fp16, one 256-byte row per thread
        // (the MMA warp commits `drain` once, after the last P V)
        if (ok && nst > 0) ok = mbar_wait_bounded(drain, 0, kWait);
        if (!ok) {
            if (lane == 0) {
                atomicOr(p.err, KV_DEV_TIMEOUT);
                abort_flag = 1;
            }
        } else {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __half* dst = p.out + (((int64_t)s * p.q_len + jbase + jr) * p.Hq + (int64_t)kvh * p.G +
                                   (r % p.G)) * D;
            for (int c0 = 0; c0 < D; c0 += 32) {
                float o32[32];
                tmem_ld32(lane_base + o_col + c0, o32);
                tmem_wait_ld();
                if (nst == 0) {  // nothing visible (context shorter than the window)
#pragma unroll
                    for (int i = 0; i < 32; ++i) o32[i] = 0.f;
                }
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v;
                        v.x = pack_half2(o32[i] * inv, o32[i + 1] * inv);
                        v.y = pack_half2(o32[i + 2] * inv, o32[i + 3] * inv);
                        v.z = pack_half2(o32[i + 4] * inv, o32[i + 5] * inv);
                        v.w = pack_half2(o32[i + 6] * inv, o32[i + 7] * inv);
                        *reinterpret_cast<uint4*>(dst + c0 + i) = v;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace pkv_prefill

// ===========================================================================
// Host side
namespace {

using namespace pkv_prefill;

PFN_cuTensorMapEncodeTiled_v12000 g_enc = nullptr;
std::mutex g_mu;

int encoder()
{
    if (g_enc) return KV_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return kv_fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    g_enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return KV_OK;
}

int encode(CUtensorMap* m, const void* base, cuuint32_t rank, const cuuint64_t* dims,
           const cuuint64_t* strides, const cuuint32_t* box)
{
    const cuuint32_t es[3] = {1, 1, 1};
    CUresult r = g_enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(base), dims, strides,
                       box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KV_OK : kv_fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled failed (prefill)");
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace {
int prefill_impl(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                 int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t q_len, float scale,
                 void* out, int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                 int32_t num_blocks, const paged_attention_opts* opts, void* stream);
}

extern "C" int paged_prefill_attention(const void* q, const void* k_pool, const void* v_pool,
                                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                                       const int32_t* context_lens, int32_t q_len, float scale,
                                       void* out, int32_t B, int32_t Hq, int32_t Hkv,
                                       int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                       void* stream)
{
    return prefill_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, q_len, scale,
                        out, B, Hq, Hkv, head_dim, block_size, num_blocks, nullptr, stream);
}

extern "C" int paged_prefill_attention_ex(const void* q, const void* k_pool, const void* v_pool,
                                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                                          const int32_t* context_lens, int32_t q_len, float scale,
                                          void* out, int32_t B, int32_t Hq, int32_t Hkv,
                                          int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                          const paged_attention_opts* opts, void* stream)
{
    return prefill_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, q_len, scale,
                        out, B, Hq, Hkv, head_dim, block_size, num_blocks, opts, stream);
}

namespace {
int prefill_impl(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                 int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t q_len, float scale,
                 void* out, int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                 int32_t num_blocks, const paged_attention_opts* opts, void* stream)
{
    if (B < 0 || q_len < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || num_blocks < 1 || max_blocks_per_seq < 1)
        return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: bad sizes");
    if (head_dim != 128) return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: head_dim must be 128");
    if (block_size != 8 && block_size != 16)
        return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: block_size must be 8 or 16");
    const int G = Hq / Hkv;
    if (G > M || M % G)
        return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: Hq/Hkv must divide 128");
    if ((uint64_t)num_blocks * Hkv * block_size >= (1ull << 31) || (uint64_t)B * q_len >= (1ull << 31))
        return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: sizes exceed 32-bit coordinates");
    if (B == 0) return KV_OK;
    if (!q || !k_pool || !v_pool || !block_tables || !context_lens || !out)
        return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: null pointer");
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_pool) || !aligned16(v_pool))
        return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: buffers must be 16-byte aligned");
    int* err = kv_error_word_ptr();
    if (!err) return kv_fail(KV_ERR_CUDA, "paged_prefill_attention: no device error word");
    int rc;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        rc = encoder();
    }
    if (rc != KV_OK) return rc;
    const int ppt = M / G;
    const int tiles = (q_len + ppt - 1) / ppt;
    const int groups = (tiles + NT - 1) / NT;  // CTAs per (sequence, kv head)
    const uint64_t grid = (uint64_t)B * Hkv * groups;
    if (grid >= (1ull << 31)) return kv_fail(KV_ERR_INVALID, "paged_prefill_attention: grid too large");
    // K / V pools as [rows][128] fp16, box = [bs rows][64 columns]
    CUtensorMap tk, tv, tq;
    const uint64_t rows = (uint64_t)num_blocks * Hkv * block_size;
    const cuuint64_t pd[2] = {(cuuint64_t)D, rows};
    const cuuint64_t ps[1] = {(cuuint64_t)D * 2};
    const cuuint32_t pb[2] = {64, (cuuint32_t)block_size};
    if ((rc = encode(&tk, k_pool, 2, pd, ps, pb)) != KV_OK) return rc;
    if ((rc = encode(&tv, v_pool, 2, pd, ps, pb)) != KV_OK) return rc;
    // q as [B*q_len positions][Hq heads][128], box = [ppt positions][G heads][64]
    const cuuint64_t qd[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)B * q_len};
    const cuuint64_t qs[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    const cuuint32_t qb[3] = {64, (cuuint32_t)G, (cuuint32_t)ppt};
    if ((rc = encode(&tq, q, 3, qd, qs, qb)) != KV_OK) return rc;

    Params prm;
    prm.q = static_cast<const __half*>(q);
    prm.out = static_cast<__half*>(out);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.err = err;
    prm.max_blocks = max_blocks_per_seq;
    prm.B = B;
    prm.q_len = q_len;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.G = G;
    prm.bs = block_size;
    prm.num_blocks = num_blocks;
    prm.tiles_per_head = groups;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.idle_ns = (opts && opts->producer_wait_ns > 0) ? (uint64_t)opts->producer_wait_ns : kWait;
    static std::mutex amu;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(amu);
        if (dev < 64 && !(configured & (1ull << dev))) {
            rc = kv_cuda_check(cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    SMEM_ALLOC),
                               "cudaFuncSetAttribute (prefill)");
            if (rc != KV_OK) return rc;
            configured |= 1ull << dev;
        }
    }
    prefill_kernel<<<(unsigned)grid, NTHREADS, SMEM_ALLOC, static_cast<cudaStream_t>(stream)>>>(tk, tv, tq,
                                                                                                prm);
    return kv_cuda_check(cudaGetLastError(), "paged_prefill_attention launch");
}

}  // namespace
