// Paged decode / verify attention for sm_100a.
//
// What is computed ("大模型推理加速与显存黑科技 (Inference Acceleration & KV Cache)"
// §2, the Attention(Q,K,V) formula): for every sequence s, window row j and
// query head h,  out = softmax(scale * q . K_t) V_t  over the visible tokens t,
// K_t / V_t read through the sequence's block table ("LLM 推理优化：KV Cache、
// PagedAttention 与量化" §2.2; the same §3.2 figure of the first page with
// 16-token blocks).  The softmax is streamed: tiles of K/V are staged on chip
// and a running maximum and denominator are kept ("大模型推理加速与显存黑科技"
// §4.2, tiling with an online softmax).  Query heads form contiguous groups
// that share one KV head ("大模型推理加速：从 KV Cache 到投机采样的工程实践"
// §"主流优化策略", GQA).  Row j of a verify window sees tokens up to
// L - q_len + j ("LLM推理优化实战：从KV Cache到Speculative Decoding" §"Speculative
// Decoding：用草稿模型加速", verify in one target pass).
//
// Design (B200):
//  * Work is the flattened space of (sequence, kv-head, block) units.  Each
//    persistent CTA takes one equal contiguous run of units, so CTAs stay
//    balanced for any length mix; a (sequence, kv-head) that straddles CTAs
//    yields partial results (o/l, log2-sum-exp) that a second kernel merges
//    (split-context log-sum-exp merge).  The schedule is computed on the
//    device from context_lens: no host planning, no per-step copies.
//  * One producer warp streams K and V tiles with 2-D TMA (128-byte swizzle)
//    into a ring of shared-memory stages (mbarrier complete_tx), plus the
//    query rows with a 1-D bulk copy at each segment start.  Consumer warps
//    take 16 tokens each of a stage: 8 warps per 128-token stage on the FMA
//    path (twice the loads in flight for its latency-bound matrix-vector
//    work), 4 warps per 64-token stage on the tensor-core paths.
//  * When the rows sharing a KV head (GQA group x window) make the products a
//    dense contraction (rows > 1), q K^T and P V run on tensor cores
//    (mma.sync m16n8k16, fp16 in, fp32 accumulate), fed by conflict-free
//    ldmatrix from the swizzled tiles.  With one row (MHA decode) the work is
//    a matrix-vector product and runs on the FMA pipes with warp shuffles.
//    An opt-in consumer computes the same on the 5th-generation tensor cores
//    (tcgen05, accumulators in tensor memory; consumer_um): at 8-24 rows per
//    KV head the contraction is too thin for it to beat the warp-level MMAs
//    (each tcgen05.mma holds its issuing thread ~95 cycles whatever its N).
//  * Every wait is bounded; a timeout or a bad block id sets a bit in the
//    device error word and the kernel returns without trapping.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/paged_kv.h"
#include "kv_device.h"
#include "kv_ptx.cuh"
#include "kv_status.h"

namespace pkv {

constexpr int kMaxMT = 2;                   // m16 tiles of rows per KV head (rows <= 32)
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kSmemBudget = 225 * 1024;
// Fixed cost of a (sequence, kv-head) segment when work is divided among CTAs,
// in tokens of K/V streaming (query load, merge, partial last stage): about
// one 128-token stage, two for int8 keys on the tensor-core path (a third
// less bytes per token, and the scaled query fragments to build)
constexpr int kSegCostTokens = 128;
constexpr int kSegCostTokensQ8 = 256;
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kRescaleThreshold = 8.f;  // log2 units: weights stay below 2^8

enum : int32_t { F_FIRST = 1, F_LAST = 2, F_WHOLE = 4, F_END = 8 };

struct StageMeta {
    int32_t s, kvh, t0, ntok, L, flags, slot, pad;
};

struct Params {
    const __half* q;
    __half* out;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* part_o;    // [grid][2][RP][D]
    float* part_lse;  // [grid][2][RP]
    int4* meta;       // [grid]: {s, kvh, first cta, slot in first cta} or s = -1
    int* err;
    const float* k_scale;  // [Hkv][D] channel scales of an int8 K pool (else null)
    int32_t max_blocks, B, q_len, Hq, Hkv, G, rows, num_blocks, min_share;
    int32_t seg_cost;  // virtual blocks charged per (sequence, kv-head) segment
    // head pairs (Hkv above counts pairs): query rows per head; padded rows
    // 8h .. 8h + pr - 1 belong to head h of the pair.  0: one head per unit.
    int32_t pr;
    float scale_log2;
    uint64_t slot_wait_ns;  // limit of the producer's waits for a free ring slot
};

// Query head and window position j of padded row R of KV head (or head pair)
// kvh; -1 for a padding row.  Row r of a head is window position r / G,
// query head g = r % G of the head's group.
__device__ __forceinline__ int row_head(const Params& p, int kvh, int R, int& j)
{
    int r = R, h0 = kvh;
    if (p.pr) {
        r = R & 7;
        h0 = 2 * kvh + (R >> 3);
        if (r >= p.pr) return -1;
    } else if (R >= p.rows) {
        return -1;
    }
    j = r / p.G;
    return h0 * p.G + r % p.G;
}

template <int D_, int BS_, int MT_, bool FMA_, bool KQ_ = false, int NR8_ = 0, int TW_ = 0,
          int SUBS_ = 1, int UMR_ = 0, int HP_ = 1>
struct Cfg {
    static constexpr int D = D_, BS = BS_, MT = MT_;
    static constexpr bool FMA = FMA_;
    static constexpr bool KQ = KQ_;  // K pool of int8 codes with per-channel scales
    // NR8 > 0: tensor-core consumer over S^T = K Q^T (tokens as the MMA's M
    // dimension, query rows as N, in NR8 tiles of 8 rows)
    static constexpr int NR8 = NR8_;
    // UMR > 0: tcgen05 consumer (accumulators in tensor memory), query rows
    // padded to UMR; each of the 128 TMEM lanes holds one query row and a
    // 128/UMR-th of the stage's tokens (see consumer_um)
    static constexpr int UMR = UMR_;
    static_assert(!UMR || (D == 128 && MT == 1 && !FMA && NR8 == 0 && SUBS_ == 1 &&
                           (UMR == 8 || UMR == 16 || UMR == 32)),
                  "the tcgen05 consumer serves head_dim 128, 8/16/32 padded rows");
    static_assert(!KQ || D == 128, "int8 K pools are served at head_dim 128");
    // HP = 2: a unit of work is a pair of adjacent KV heads of a block, staged
    // by one copy of both heads' rows (they are contiguous in the pool): half
    // the copies per byte.  Row tile h holds the query rows of head h of the
    // pair (padded rows 8h .., at most 8 per head; see row_head).
    static constexpr int HP = HP_;
    static_assert(HP == 1 || (HP == 2 && NR8_ == 2 && !UMR && D == 128),
                  "head pairs: two row tiles of one head each, head_dim 128");
    static constexpr int NH = D / 64;                       // 64-column halves per row
    // consumer warps along the tokens of a stage (16 tokens each) and tokens
    // per stage: the FMA consumers run latency-bound matrix-vector work and
    // gain from twice the warps; the tensor-core consumers keep 4 (with 9
    // warps their register cap would drop to 168 and the merge at each
    // segment end would take twice the rounds)
    static constexpr int TW = UMR ? 8 : (TW_ ? TW_ : (FMA ? 8 : 4));
    // 16-token sub-tiles each consumer warp takes per stage (the transposed
    // tensor-core consumer only): larger stages at the same register count
    static constexpr int SUBS = SUBS_;
    static_assert(SUBS == 1 || NR8 > 0, "sub-tiles need the transposed consumer");
    static constexpr int TS = 16 * TW * SUBS;               // tokens per pipeline stage
    static_assert(TS / BS <= 32, "one producer lane per block of a stage");
    static constexpr int NBS = TS / BS;                     // blocks per stage
    static constexpr int RP = UMR ? UMR : (FMA ? 1 : (NR8 ? 8 * NR8 : 16 * MT));  // padded rows
    // consumer warps (the tcgen05 consumer: 4 softmax warps, one per TMEM
    // lane quarter, plus the MMA-issuing warp after the producer)
    static constexpr int NCW = UMR ? 4 : TW;
    static constexpr int THREADS = (NCW + (UMR ? 2 : 1)) * 32;
    // registers per thread for one CTA per SM: warps are spread over the 4
    // SM sub-partitions, each with a 16K-register file
    static constexpr int WARPS_PER_SUBPART = (THREADS / 32 + 3) / 4;
    static constexpr int MAXREG_RAW = (16384 / (32 * WARPS_PER_SUBPART)) / 8 * 8;
    static constexpr int MAXREG = MAXREG_RAW > 255 ? 255 : MAXREG_RAW;
    static constexpr int TROWS = BS * HP;                   // pool rows of one staged tile
    static constexpr int TILE_BYTES = TROWS * D * 2;        // one (block, kv-head[s]) fp16 tile
    static constexpr int KV_BYTES = TS * HP * D * 2;        // fp16 K (or V) bytes per stage
    static constexpr int K_TILE_BYTES = KQ ? TROWS * D : TILE_BYTES;
    // the tcgen05 consumer keeps fp16 room for K also over int8 codes: they
    // land in its upper half and are widened in place
    static constexpr int K_BYTES = (KQ && !UMR) ? TS * HP * D : KV_BYTES;
    // one 64-column half of a stage's K or V in the tcgen05 consumer's layout
    // ([half][token][128 B], the MMA's 128-byte-swizzle K-major / MN-major form)
    static constexpr int UM_HALF = TS * 128;
    static constexpr int V_OFF = K_BYTES;                   // stage: K, V, query rows
    // query rows of a segment, one per 16-byte-padded row (conflict-free ldmatrix)
    static constexpr int QROW = D * 2 + 16;
    static constexpr int Q_BYTES = (RP * QROW + (KQ ? HP * D * 4 : 0) + 1023) / 1024 * 1024;
    static constexpr int Q_OFF = K_BYTES + KV_BYTES;
    // int8 keys: the segment's channel scales (D fp32 per head) follow the query rows
    static constexpr int SC_OFF = Q_OFF + RP * QROW;
    static_assert(!KQ || RP * QROW + HP * D * 4 <= Q_BYTES, "room for the channel scales");
    static constexpr int STAGE_BYTES = Q_OFF + Q_BYTES;
    // floats per obuf row (the transposed consumer's scalar stores of rows
    // 2*tig, 2*tig+1 are conflict-free when 2 * OB_STRIDE = 8 mod 32)
    static constexpr int OB_STRIDE = NR8 ? D + 4 : D + 8;
    static constexpr int OBUF_SLICE = RP * OB_STRIDE;               // floats
    // two merge slices (the transposed consumer merges in the stage it just
    // consumed instead: one slice per token warp, see consumer_tc)
    static constexpr int OBUF_BYTES = (NR8 || UMR) ? 0 : 2 * OBUF_SLICE * 4;
    static constexpr int ML_BYTES = UMR ? 128 * 2 * 4 : TW * RP * 2 * 4;
    // CTA copy of the query rows (read again every stage)
    static constexpr bool QPERSIST = UMR ? false : (NR8 ? NR8 > 2 : MT > 1);
    // rows of that copy: whole pairs of 8-row tiles (B fragments of two row
    // tiles come from one ldmatrix)
    static constexpr int QP_ROWS = NR8 ? 16 * ((NR8 + 1) / 2) : RP;
    static constexpr int QP_BYTES = QPERSIST ? QP_ROWS * QROW : 0;
    static constexpr int UM_NBARS = UMR ? 12 : 0;  // the tcgen05 consumer's barriers
    static constexpr int FIXED = OBUF_BYTES + ML_BYTES + QP_BYTES + 256 + 16 * 64 + UM_NBARS * 8 + 16;
    static constexpr int STAGES_RAW = (kSmemBudget - FIXED) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static_assert(STAGES >= 2, "not enough shared memory for two stages");
    static constexpr int META_OFF = STAGES * STAGE_BYTES;   // StageMeta[STAGES]
    static constexpr int BAR_OFF = META_OFF + STAGES * 32;  // full[S], empty[S]
    static constexpr int ZERO_OFF = BAR_OFF + STAGES * 16;  // 128 zero bytes
    static constexpr int PB_OFF = ZERO_OFF + 128;           // per-warp fp16 weights (FMA path)
    static constexpr int ML_OFF = PB_OFF + TW * 32;
    static constexpr int OBUF_OFF = ML_OFF + ML_BYTES;
    static constexpr int QP_OFF = OBUF_OFF + OBUF_BYTES;
    static constexpr int UB_OFF = QP_OFF + QP_BYTES;        // tcgen05 consumer barriers
    static constexpr int TSLOT_OFF = UB_OFF + UM_NBARS * 8; // its tensor-memory base address
    static constexpr int SMEM_USED = TSLOT_OFF + (UMR ? 16 : 0);
    static_assert(!UMR || 128 * D * 4 <= Q_OFF, "the segment-end slices fit a stage's K and V");
    // merge slices at a segment end: one per token warp, or, when TW of them
    // do not fit a stage, one per pair of warps (w and w + TW/2, added in place)
    static constexpr int MSLOTS = (NR8 && TW * OBUF_SLICE * 4 > STAGE_BYTES) ? TW / 2 : TW;
    static_assert(!NR8 || MSLOTS * OBUF_SLICE * 4 <= STAGE_BYTES, "merge slices fit a stage");
    static constexpr int SMEM_ALLOC = SMEM_USED + 1024;    // room to align the base
};

__device__ __forceinline__ int32_t nblk_of(int32_t L, int32_t bs, int32_t max_blocks)
{
    int32_t nb = L <= 0 ? 1 : (L + bs - 1) / bs;
    return nb > max_blocks ? max_blocks : nb;
}

__device__ __forceinline__ int32_t clamp_len(int32_t L, int32_t bs, int32_t max_blocks)
{
    if (L < 0) return 0;
    const int32_t cap = max_blocks * bs;
    return L > cap ? cap : L;
}

__device__ __forceinline__ int64_t warp_sum64(int64_t v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int64_t warp_incl_scan64(int64_t v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int64_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Shared-memory layout of a staged tile: one (block, kv-head) tile is its
// BS rows of D fp16, i.e. BS * NH units of 128 bytes in global order (one TMA
// copy of the contiguous tile).  The 128-byte swizzle stores 16-byte chunk c
// of unit u at chunk position c ^ (u mod 8).  A head pair's tile is head 0's
// BS rows, then head 1's.  Byte offset, inside a stage's K (or V) area, of
// chunk cg (0 .. D/8-1) of stage token `tok` of head h of the tile:
template <class C>
__device__ __forceinline__ uint32_t tile_chunk(int tok, int cg, int h = 0)
{
    const int r = h * C::BS + tok % C::BS;  // row of head h of the pair
    const int u = r * C::NH + (cg >> 3);
    return (uint32_t)((tok / C::BS) * C::TILE_BYTES + u * 128 + (((cg & 7) ^ (u & 7)) << 4));
}

// The same for an int8 K tile: one 128-byte unit (D = 128 codes) per token.
template <class C>
__device__ __forceinline__ uint32_t tile_chunk_k8(int tok, int cg, int h = 0)
{
    const int r = h * C::BS + tok % C::BS;
    return (uint32_t)((tok / C::BS) * C::K_TILE_BYTES + r * 128 + ((cg ^ (r & 7)) << 4));
}

// q times the channel scales of an int8 K pool (fp16 pair, round to nearest).
__device__ __forceinline__ uint32_t scale_h2(uint32_t h2, float2 sc)
{
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    return pack_half2(f.x * sc.x, f.y * sc.y);
}

// int8 codes -> fp16: the byte x + 128 (x ^ 0x80) becomes the low mantissa
// byte of an fp16 with exponent byte 0x64, whose value is 1024 + x + 128
// exactly (1152 + x).

// Biased form used on the hot path: four codes -> two half2 holding
// 1152 + code exactly (no subtraction).  A dot product over biased keys
// exceeds the true one by 1152 * (sum of the q entries), a per-row constant
// subtracted once per score.
__device__ __forceinline__ void i8x4_to_h2x2_biased(uint32_t w, uint32_t& lo, uint32_t& hi)
{
    const uint32_t u = w ^ 0x80808080u;
    asm("prmt.b32 %0, %1, %2, 0x5140;" : "=r"(lo) : "r"(u), "r"(0x64646464u));
    asm("prmt.b32 %0, %1, %2, 0x7362;" : "=r"(hi) : "r"(u), "r"(0x64646464u));
}
constexpr float kCodeBias = 1152.f;

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float h2_sum(uint32_t h2)
{
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    return f.x + f.y;
}

// B fragments of k-step ks for the two n8 tiles (tokens t0 and t0 + 8) from an
// int8 K stage, biased.  The dims of each 16-dim chunk are taken in a
// permuted order, so that one 32-bit word per token serves both registers:
// lane tig's k positions (2tig, 2tig+1 | 2tig+8, 2tig+9) are dims
// (4tig, 4tig+1 | 4tig+2, 4tig+3); the q fragments use the same order.
template <class C>
__device__ __forceinline__ void k8_frag(uint32_t st, int t0, int ks, int tig, uint32_t& b0,
                                        uint32_t& b1, uint32_t& b2, uint32_t& b3)
{
    i8x4_to_h2x2_biased(lds_u32(st + tile_chunk_k8<C>(t0, ks) + 4 * tig), b0, b1);
    i8x4_to_h2x2_biased(lds_u32(st + tile_chunk_k8<C>(t0 + 8, ks) + 4 * tig), b2, b3);
}

// One TMA copy of the tile whose first row is `y` in the pool's row space.
template <int NH>
__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap* tm, int32_t y,
                                              uint32_t bar, uint64_t pol)
{
    if constexpr (NH == 1)
        tma_load_2d(dst, tm, 0, y, bar, pol);
    else
        tma_load_3d(dst, tm, 0, 0, y, bar, pol);
}

// ---------------------------------------------------------------------------
// Producer warp: walks this CTA's run of units and feeds the stage ring.
//
// Block-table entries are loaded one batch of kLA stages ahead of the stage
// being issued, so the table's load latency overlaps the copies in flight
// instead of sitting in front of every TMA issue.
constexpr int kLA = 4;  // stages per look-ahead batch

struct StageDesc {
    int32_t s, kvh, b, nbl, t0, ntok, L, flags, slot;
};

// Walks (sequence, kv-head, block) units of one CTA's run and cuts them into
// stages of at most NBS blocks that never cross a (sequence, kv-head).
template <class C>
struct UnitWalker {
    const Params* p;
    int lane;
    int64_t u, u1, share, seq_start;
    int32_t s, L, nb;
    int32_t kvh, b, b1, slot;
    bool whole, in_seg, first_seg, seg_first_stage;
    int32_t win_base, win_len;  // lane i holds context_lens[win_base + i]
    int4 merge_meta;            // what the merge kernel needs from this CTA

    __device__ int32_t len_of(int32_t seq)
    {
        if (seq >= win_base + 32 || seq < win_base) {
            win_base = seq;
            win_len = seq + lane < p->B ? __ldg(p->context_lens + seq + lane) : 0;
        }
        return __shfl_sync(0xffffffffu, win_len, seq - win_base);
    }

    __device__ void enter_sequence(int32_t seq)
    {
        s = seq;
        const int32_t Lraw = len_of(seq);
        L = clamp_len(Lraw, C::BS, p->max_blocks);
        nb = nblk_of(Lraw, C::BS, p->max_blocks);
        if (lane == 0 && Lraw > L) atomicOr(p->err, KV_DEV_BAD_BLOCK);
    }

    // Next stage of the run; false when the run is exhausted.
    // Each (sequence, kv-head) spans seg_cost virtual units (its fixed cost:
    // query load, merge, partial last stage) followed by its nb blocks, so
    // equal runs of units also even out the number of segments per CTA.
    __device__ bool next(StageDesc& d)
    {
        if (!in_seg) {
            if (u >= u1) return false;
            const int64_t span = (int64_t)nb + p->seg_cost;
            const int64_t local = u - seq_start;
            kvh = (int32_t)(local / span);
            const int64_t off = local % span;
            if (off < p->seg_cost) {  // skip the virtual units
                u += p->seg_cost - off;
                if (u >= u1) return false;
            }
            b = (int32_t)((u - seq_start) % span - p->seg_cost);
            const int64_t kv_end = seq_start + (int64_t)(kvh + 1) * span;
            const int64_t seg_end = u1 < kv_end ? u1 : kv_end;
            b1 = b + (int32_t)(seg_end - u);
            whole = b == 0 && b1 == nb;
            slot = first_seg ? 0 : 1;
            if (first_seg && b > 0 && b1 == nb) {
                // first CTA of this (sequence, kv-head): the one holding its
                // first block; its piece is that CTA's first segment exactly
                // when the CTA's run starts at or after the virtual units
                const int64_t gstart = seq_start + (int64_t)kvh * span + p->seg_cost;
                const int64_t a = gstart / share;
                merge_meta = make_int4(s, kvh, (int32_t)a, a * share >= gstart - p->seg_cost ? 0 : 1);
            }
            first_seg = false;
            in_seg = true;
            seg_first_stage = true;
        }
        const int32_t nbl = (b1 - b) < C::NBS ? (b1 - b) : C::NBS;
        d.s = s;
        d.kvh = kvh;
        d.b = b;
        d.nbl = nbl;
        d.t0 = b * C::BS;
        int32_t tend = (b + nbl) * C::BS;
        if (tend > L) tend = L;
        d.ntok = tend > d.t0 ? tend - d.t0 : 0;
        d.L = L;
        d.flags = (seg_first_stage ? F_FIRST : 0) | (b + nbl >= b1 ? F_LAST : 0) |
                  (whole ? F_WHOLE : 0);
        d.slot = slot;
        seg_first_stage = false;
        b += nbl;
        u += nbl;
        if (b >= b1) {
            in_seg = false;
            if (u < u1 && u == seq_start + ((int64_t)nb + p->seg_cost) * p->Hkv) {
                seq_start = u;
                enter_sequence(s + 1);
            }
        }
        return true;
    }
};

// Work units of sequence s: (blocks + the per-segment cost) x KV heads.
template <class C>
__device__ __forceinline__ int64_t units_of(const Params& p, int32_t Lraw)
{
    return ((int64_t)nblk_of(Lraw, C::BS, p.max_blocks) + p.seg_cost) * p.Hkv;
}

template <class C>
__device__ void producer(const CUtensorMap* tmK, const CUtensorMap* tmV, const Params& p,
                         uint8_t* smem, volatile int* abort_flag)
{
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    StageMeta* smeta = reinterpret_cast<StageMeta*>(smem + C::META_OFF);
    const uint32_t full0 = sbase + C::BAR_OFF;
    const uint32_t empty0 = full0 + C::STAGES * 8;
    const uint64_t pol = l2_policy_evict_first();
    if (lane == 0) {
        prefetch_tmap(tmK);
        prefetch_tmap(tmV);
    }
    // Each CTA pulls an equal slice of the block tables into L2 while it
    // scans the lengths, so the table reads that follow the scan (by
    // whichever CTA) hit L2 instead of waiting on DRAM (and its page walk).
    {
        const uint64_t tbytes = (uint64_t)p.B * (uint64_t)p.max_blocks * 4u;
        uint64_t chunk = (tbytes + gridDim.x - 1) / gridDim.x;
        chunk = (chunk + 127) / 128 * 128;
        if (chunk > 65536) chunk = 65536;
        const uint64_t begin = (uint64_t)blockIdx.x * chunk;
        const char* tb = reinterpret_cast<const char*>(p.block_tables);
        for (uint64_t off = begin + (uint64_t)lane * 128; off < begin + chunk && off < tbytes; off += 32 * 128)
            prefetch_l2(tb + off);
    }

    // Pass 1: total units.  Each lane takes 8 consecutive sequences of a
    // 256-sequence chunk; all loads of a chunk are in flight together.
    int64_t total = 0;
    for (int base = 0; base < p.B; base += 256) {
        int64_t sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int s = base + lane * 8 + j;
            if (s < p.B) sum += units_of<C>(p, __ldg(p.context_lens + s));
        }
        total += warp_sum64(sum);
    }
    const int64_t G = gridDim.x;
    int64_t share = (total + G - 1) / G;
    if (share < p.min_share) share = p.min_share;
    const int64_t u0 = (int64_t)blockIdx.x * share;
    const int64_t u1 = u0 + share < total ? u0 + share : total;

    UnitWalker<C> w;
    w.p = &p;
    w.lane = lane;
    w.merge_meta = make_int4(-1, 0, 0, 0);
    w.win_base = -64;
    w.win_len = 0;
    bool ok = true;
    int k_issued = 0;  // stages issued so far (the end marker included)
    // Wait for ring slot `stage` to be free again (its previous use, `round`
    // - 1, consumed).  Every lane waits; lane 0's outcome (and its reading of
    // the abort flag) decides for the warp, so the lanes never disagree.
    auto slot_wait = [&](int stage, int round, uint64_t limit) -> bool {
        const uint32_t bar = empty0 + stage * 8;
        const uint32_t par = (uint32_t)(round - 1) & 1u;
        bool got = limit >= kWaitLimitNs ? mbar_wait_bounded(bar, par, limit)
                                         : mbar_wait_fine(bar, par, limit);
        got = got && !*abort_flag;
        return __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
    };

    if (u0 < u1) {
        // Pass 2: the sequence holding unit u0.
        int s0 = -1;
        int64_t start0 = 0, run = 0;
        for (int base = 0; base < p.B && s0 < 0; base += 256) {
            int64_t uu[8];
            int64_t sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int s = base + lane * 8 + j;
                uu[j] = s < p.B ? units_of<C>(p, __ldg(p.context_lens + s)) : 0;
                sum += uu[j];
            }
            const int64_t incl = warp_incl_scan64(sum, lane);
            const int64_t excl = run + incl - sum;
            const bool hit = excl <= u0 && u0 < excl + sum;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            if (m) {
                const int src = __ffs(m) - 1;
                int64_t acc = excl;
                int found = -1;
                int64_t fstart = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (found < 0 && uu[j] > 0 && acc <= u0 && u0 < acc + uu[j]) {
                        found = base + lane * 8 + j;
                        fstart = acc;
                    }
                    acc += uu[j];
                }
                s0 = __shfl_sync(0xffffffffu, found, src);
                start0 = __shfl_sync(0xffffffffu, fstart, src);
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (s0 < 0) {  // unreachable when u0 < total; keeps the walk well defined
            s0 = 0;
            ok = false;
        }
        w.u = u0;
        w.u1 = ok ? u1 : u0;
        w.share = share;
        w.seq_start = start0;
        w.in_seg = false;
        w.first_seg = true;
        w.seg_first_stage = false;
        w.enter_sequence(s0);

        // block id of block `lane` of a stage (-1: nothing to load)
        auto load_id = [&](const StageDesc& d) -> int32_t {
            if (lane < d.nbl && d.t0 + lane * C::BS < d.L)
                return __ldg(p.block_tables + (int64_t)d.s * p.max_blocks + d.b + lane);
            return -1;
        };
        StageDesc cur[kLA], nxt[kLA];
        int32_t cid[kLA], nid[kLA];
        int ncur = 0, nnxt = 0;
#pragma unroll
        for (int k = 0; k < kLA; ++k)
            if (ncur == k && w.next(cur[k])) {
                cid[k] = load_id(cur[k]);
                ++ncur;
            }
#pragma unroll
        for (int k = 0; k < kLA; ++k)
            if (nnxt == k && w.next(nxt[k])) {
                nid[k] = load_id(nxt[k]);
                ++nnxt;
            }
        // Everything above reads only the lengths and block tables; the pools
        // (and q) may still be being written by the grid this launch depends
        // on (a cache append launched just before): wait for it here.
        pdl_wait();
        while (ncur > 0 && ok) {
#pragma unroll
            for (int k = 0; k < kLA; ++k) {
                if (k >= ncur || !ok) break;
                const StageDesc& d = cur[k];
                const int stage = k_issued % C::STAGES;
                const int round = k_issued / C::STAGES;
                if (round > 0 && !slot_wait(stage, round, p.slot_wait_ns)) {
                    ok = false;
                    break;
                }
                const int32_t id = cid[k];
                const bool has_tok = lane < d.nbl && d.t0 + lane * C::BS < d.L;
                const bool bad = has_tok && (id < 0 || id >= p.num_blocks);
                const bool load = has_tok && !bad;
                const unsigned lmask = __ballot_sync(0xffffffffu, load);
                if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err, KV_DEV_BAD_BLOCK);
                const bool firstst = (d.flags & F_FIRST) != 0;
                const uint32_t qbytes = (uint32_t)(p.G * C::D * 2) * (p.pr ? 2u : 1u);  // per window row
                uint32_t bytes = (uint32_t)__popc(lmask) * (uint32_t)(C::K_TILE_BYTES + C::TILE_BYTES);
                if (firstst) bytes += qbytes * (uint32_t)p.q_len + (C::KQ ? C::HP * C::D * 4 : 0);
                const uint32_t full = full0 + stage * 8;
                if (lane == 0) {
                    StageMeta& md = smeta[stage];
                    md.s = d.s;
                    md.kvh = d.kvh;
                    md.t0 = d.t0;
                    md.ntok = d.ntok;
                    md.L = d.L;
                    md.flags = d.flags;
                    md.slot = d.slot;
                    mbar_arrive_expect_tx(full, bytes);
                }
                __syncwarp();
                const uint32_t st = sbase + stage * C::STAGE_BYTES;
                if (load) {
                    const int32_t y = (id * p.Hkv + d.kvh) * C::TROWS;
                    if constexpr (C::UMR > 0) {
                        // block `lane` -> rows [lane*BS, lane*BS+BS) of each 64-column
                        // half; int8 codes (128 per row) into the upper half of K
                        const uint32_t ko = st + (uint32_t)(lane * C::BS * 128);
                        if constexpr (C::KQ) {
                            tma_load_2d(ko + C::UM_HALF, tmK, 0, y, full, pol);
                        } else {
                            tma_load_2d(ko, tmK, 0, y, full, pol);
                            tma_load_2d(ko + C::UM_HALF, tmK, 64, y, full, pol);
                        }
                        tma_load_2d(ko + C::V_OFF, tmV, 0, y, full, pol);
                        tma_load_2d(ko + C::V_OFF + C::UM_HALF, tmV, 64, y, full, pol);
                    } else {
                        if constexpr (C::KQ)
                            tma_load_2d(st + (uint32_t)(lane * C::K_TILE_BYTES), tmK, 0, y, full, pol);
                        else
                            tma_load_tile<C::NH>(st + (uint32_t)(lane * C::TILE_BYTES), tmK, y, full, pol);
                        tma_load_tile<C::NH>(st + C::V_OFF + (uint32_t)(lane * C::TILE_BYTES), tmV, y,
                                             full, pol);
                    }
                }
                int qj = 0;
                const int qh = (firstst && lane < p.rows) ? row_head(p, d.kvh, lane, qj) : -1;
                if (qh >= 0) {  // padded row `lane` of the segment's queries
                    const __half* src = p.q + (((int64_t)d.s * p.q_len + qj) * p.Hq + qh) * C::D;
                    bulk_load(st + C::Q_OFF + lane * C::QROW, src, C::D * 2, full);
                }
                if (C::KQ && firstst && lane == 31)  // the KV head's (pair's) channel scales
                    bulk_load(st + C::SC_OFF, p.k_scale + (int64_t)d.kvh * C::HP * C::D, C::HP * C::D * 4,
                              full);
                ++k_issued;
            }
#pragma unroll
            for (int k = 0; k < kLA; ++k) {
                cur[k] = nxt[k];
                cid[k] = nid[k];
            }
            ncur = nnxt;
            nnxt = 0;
#pragma unroll
            for (int k = 0; k < kLA; ++k)
                if (nnxt == k && w.next(nxt[k])) {
                    nid[k] = load_id(nxt[k]);
                    ++nnxt;
                }
        }
    }
    if (lane == 0) p.meta[blockIdx.x] = w.merge_meta;

    // End marker, also after giving up: the consumers then finish the stages
    // already issued and stop at the marker instead of waiting out their own
    // limit on a stage that never comes.  After a give-up the slot wait uses
    // the full limit (the consumers are still draining the ring), unless a
    // consumer has already stopped.
    {
        const int stage = k_issued % C::STAGES;
        const int round = k_issued / C::STAGES;
        bool slot_ok = round == 0;
        if (!slot_ok && ok) slot_ok = slot_wait(stage, round, p.slot_wait_ns);
        if (!slot_ok) ok = false;
        if (!slot_ok) slot_ok = slot_wait(stage, round, kWaitLimitNs);
        if (slot_ok) {
            if (lane == 0) {
                smeta[stage].flags = F_END;
                mbar_arrive(full0 + stage * 8);
            }
            ++k_issued;
        }
    }
    if (!ok) {
        if (lane == 0) {
            atomicOr(p.err, KV_DEV_TIMEOUT);
            *abort_flag = 1;
        }
    }
    // Drain: every issued stage's copies must have landed before the CTA may
    // exit (consumers normally wait for them anyway).
    for (int i = lane; i < C::STAGES && i < k_issued; i += 32) {
        const int n_i = (k_issued - i + C::STAGES - 1) / C::STAGES;  // issues into slot i
        if (!mbar_wait_bounded(full0 + i * 8, (n_i - 1) & 1, kWaitLimitNs))
            atomicOr(p.err, KV_DEV_TIMEOUT);
    }
}

// ---------------------------------------------------------------------------
// Output of a finished segment: the two `obuf` slices hold the token-warps'
// rescaled o (summed here, always in the same order); `mlb` holds per
// token-warp (m, l).  Writes fp16 output or fp32 partials.
template <class C>
__device__ void store_segment(const Params& p, const StageMeta& md, const float* obuf,
                              const float* mlb, int tid)
{
    const int rows = p.rows;
    if (md.flags & F_WHOLE) {
        for (int idx = tid; idx < rows * (C::D / 8); idx += C::NCW * 32) {
            const int R = idx / (C::D / 8);
            const int d0 = (idx % (C::D / 8)) * 8;
            const int j = R / p.G, g = R % p.G;
            const float4* a = reinterpret_cast<const float4*>(obuf + R * C::OB_STRIDE + d0);
            const float4* b = reinterpret_cast<const float4*>(obuf + C::OBUF_SLICE + R * C::OB_STRIDE + d0);
            const float4 a0 = a[0], a1 = a[1], b0 = b[0], b1 = b[1];
            uint4 v;
            v.x = pack_half2(a0.x + b0.x, a0.y + b0.y);
            v.y = pack_half2(a0.z + b0.z, a0.w + b0.w);
            v.z = pack_half2(a1.x + b1.x, a1.y + b1.y);
            v.w = pack_half2(a1.z + b1.z, a1.w + b1.w);
            __half* dst = p.out + (((int64_t)md.s * p.q_len + j) * p.Hq + (int64_t)md.kvh * p.G + g) *
                                      C::D + d0;
            *reinterpret_cast<uint4*>(dst) = v;
        }
    } else {
        const int64_t pbase = ((int64_t)blockIdx.x * 2 + md.slot) * C::RP;
        for (int idx = tid; idx < rows * (C::D / 8); idx += C::NCW * 32) {
            const int R = idx / (C::D / 8);
            const int d0 = (idx % (C::D / 8)) * 8;
            const float4* a = reinterpret_cast<const float4*>(obuf + R * C::OB_STRIDE + d0);
            const float4* b = reinterpret_cast<const float4*>(obuf + C::OBUF_SLICE + R * C::OB_STRIDE + d0);
            const float4 a0 = a[0], a1 = a[1], b0 = b[0], b1 = b[1];
            float4* dst = reinterpret_cast<float4*>(p.part_o + (pbase + R) * C::D + d0);
            dst[0] = make_float4(a0.x + b0.x, a0.y + b0.y, a0.z + b0.z, a0.w + b0.w);
            dst[1] = make_float4(a1.x + b1.x, a1.y + b1.y, a1.z + b1.z, a1.w + b1.w);
        }
        for (int R = tid; R < rows; R += C::NCW * 32) {
            float M = kNegInf;
#pragma unroll
            for (int w = 0; w < C::TW; ++w) M = fmaxf(M, mlb[(w * C::RP + R) * 2]);
            const float Mu = M == kNegInf ? 0.f : M;
            float Ls = 0.f;
#pragma unroll
            for (int w = 0; w < C::TW; ++w)
                Ls += mlb[(w * C::RP + R) * 2 + 1] * ex2(mlb[(w * C::RP + R) * 2] - Mu);
            p.part_lse[pbase + R] = Ls > 0.f ? Mu + lg2(Ls) : kNegInf;
        }
    }
}

// Output of a finished segment from TW per-warp slices (each warp's o
// already scaled by its factor), summed in warp order (bit-reproducible):
// fp16 output (whole segment) or fp32 partials.
template <class C>
__device__ void store_segment_slices(const Params& p, const StageMeta& md, const float* slices,
                                     const float* mlb, int tid)
{
    const int rows = p.rows;
    const bool whole = (md.flags & F_WHOLE) != 0;
    const int64_t pbase = ((int64_t)blockIdx.x * 2 + md.slot) * C::RP;
    for (int idx = tid; idx < rows * (C::D / 8); idx += C::NCW * 32) {
        const int R = idx / (C::D / 8);
        const int d0 = (idx % (C::D / 8)) * 8;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
#pragma unroll
        for (int w = 0; w < C::MSLOTS; ++w) {
            const float4* src = reinterpret_cast<const float4*>(slices + (w * C::RP + R) * C::OB_STRIDE + d0);
            const float4 x = src[0], y = src[1];
            a = make_float4(a.x + x.x, a.y + x.y, a.z + x.z, a.w + x.w);
            b = make_float4(b.x + y.x, b.y + y.y, b.z + y.z, b.w + y.w);
        }
        if (whole) {
            int j = 0;
            const int qh = row_head(p, md.kvh, R, j);
            if (qh < 0) continue;
            uint4 v;
            v.x = pack_half2(a.x, a.y);
            v.y = pack_half2(a.z, a.w);
            v.z = pack_half2(b.x, b.y);
            v.w = pack_half2(b.z, b.w);
            __half* dst = p.out + (((int64_t)md.s * p.q_len + j) * p.Hq + qh) * C::D + d0;
            *reinterpret_cast<uint4*>(dst) = v;
        } else {
            float4* dst = reinterpret_cast<float4*>(p.part_o + (pbase + R) * C::D + d0);
            dst[0] = a;
            dst[1] = b;
        }
    }
    if (!whole) {
        for (int R = tid; R < rows; R += C::NCW * 32) {
            float M = kNegInf;
#pragma unroll
            for (int w = 0; w < C::TW; ++w) M = fmaxf(M, mlb[(w * C::RP + R) * 2]);
            const float Mu = M == kNegInf ? 0.f : M;
            float Ls = 0.f;
#pragma unroll
            for (int w = 0; w < C::TW; ++w)
                Ls += mlb[(w * C::RP + R) * 2 + 1] * ex2(mlb[(w * C::RP + R) * 2] - Mu);
            p.part_lse[pbase + R] = Ls > 0.f ? Mu + lg2(Ls) : kNegInf;
        }
    }
}

// Combine the token-warps' (m, l) for row R; returns this warp's factor
// 2^(m_w - M) / sum.
template <class C>
__device__ __forceinline__ float row_factor(const float* mlb, int R, float m_w)
{
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < C::TW; ++w) M = fmaxf(M, mlb[(w * C::RP + R) * 2]);
    const float Mu = M == kNegInf ? 0.f : M;
    float Ls = 0.f;
#pragma unroll
    for (int w = 0; w < C::TW; ++w)
        Ls += mlb[(w * C::RP + R) * 2 + 1] * ex2(mlb[(w * C::RP + R) * 2] - Mu);
    return Ls > 0.f ? ex2(m_w - Mu) / Ls : 0.f;
}

// ---------------------------------------------------------------------------
// FMA consumer: one query row per KV head (MHA decode), a matrix-vector
// product, so no tensor cores.  q . k: the 8 lanes of group g = lane / 8 each
// take one 16-byte chunk per 128-byte unit of the rows of tokens g, g+4, g+8,
// g+12 (a warp-wide 16-byte load reads whole units: no bank conflicts), then
// sum over the group with shuffles.  P V: lane = D/32 output columns; the
// fp16 weights of the warp's 16 tokens are broadcast through shared memory.
template <class C>
__device__ void consumer_fma(const Params& p, uint8_t* smem, volatile int* abort_flag)
{
    constexpr int D = C::D;
    constexpr int NH = C::NH;
    constexpr int DPT = D / 32;  // P V columns per lane
    const int cw = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qw = cw;
    const uint32_t sbase = smem_u32(smem);
    const StageMeta* smeta = reinterpret_cast<const StageMeta*>(smem + C::META_OFF);
    const uint32_t full0 = sbase + C::BAR_OFF;
    const uint32_t empty0 = full0 + C::STAGES * 8;
    float* mlb = reinterpret_cast<float*>(smem + C::ML_OFF);
    float* obuf = reinterpret_cast<float*>(smem + C::OBUF_OFF);
    __half* pbuf = reinterpret_cast<__half*>(smem + C::PB_OFF) + qw * 16;
    const float sl2 = p.scale_log2;

    const int c = lane & 7, grp = lane >> 3;
    // chunk c of each unit of tokens grp + 4i; int8 keys: one 128-byte unit
    // per token, chunk c = dims 16c .. 16c+15
    uint32_t koff[4][NH];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int h = 0; h < NH; ++h)
            koff[i][h] = C::KQ ? tile_chunk_k8<C>(qw * 16 + grp + 4 * i, c)
                               : tile_chunk<C>(qw * 16 + grp + 4 * i, h * 8 + c);
    const int v_col = lane * DPT;
    const int v_cg = v_col / 8;          // chunk holding my output columns
    const int v_byte = (v_col % 8) * 2;  // byte offset inside that chunk

    uint32_t qh[NH][4];  // q columns h*64 + c*8 .. +8 (int8 keys: 16c + 8h ..) as fp16 pairs
    float corr = 0.f;    // int8 keys: bias * sum of this lane's q entries
    float o[DPT];
    float m = kNegInf, l = 0.f;

    int stage = 0;
    uint32_t phase = 0;
    for (;;) {
        if (!mbar_wait_bounded(full0 + stage * 8, phase, kWaitLimitNs)) {
            *abort_flag = 1;
            break;
        }
        const StageMeta md = smeta[stage];
        if (md.flags & F_END) break;
        const uint8_t* st = smem + stage * C::STAGE_BYTES;
        if (md.flags & F_FIRST) {
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const int d0 = C::KQ ? 16 * c + 8 * h : h * 64 + c * 8;
                const uint4 v = *reinterpret_cast<const uint4*>(st + C::Q_OFF + d0 * 2);
                qh[h][0] = v.x;
                qh[h][1] = v.y;
                qh[h][2] = v.z;
                qh[h][3] = v.w;
                if constexpr (C::KQ) {  // fold the channel scales of the int8 keys into q
                    const float* sc = reinterpret_cast<const float*>(st + C::SC_OFF) + d0;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        qh[h][e] = scale_h2(qh[h][e], *reinterpret_cast<const float2*>(sc + 2 * e));
                }
            }
            if constexpr (C::KQ) {  // bias correction of this lane's 16 dims
                float qs = 0.f;
#pragma unroll
                for (int h = 0; h < NH; ++h)
#pragma unroll
                    for (int e = 0; e < 4; ++e) qs += h2_sum(qh[h][e]);
                corr = kCodeBias * qs;
            }
#pragma unroll
            for (int i = 0; i < DPT; ++i) o[i] = 0.f;
            m = kNegInf;
            l = 0.f;
        }
        const int nv = md.ntok - qw * 16;
        if (nv > 0) {
            // partial dots of tokens grp + 4i over my chunk of every unit
            float acc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float a0 = 0.f, a1 = 0.f;
                if constexpr (C::KQ) {
                    // 16 codes: dims 16c .. 16c+15 <-> qh[0] (first 8), qh[1]
                    const uint4 kv = *reinterpret_cast<const uint4*>(st + koff[i][0]);
                    const uint32_t kw8[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint32_t lo, hi;
                        i8x4_to_h2x2_biased(kw8[w], lo, hi);
                        const uint32_t qa_ = qh[w >> 1][(w & 1) * 2], qb_ = qh[w >> 1][(w & 1) * 2 + 1];
                        a0 = fma_h((uint16_t)(qa_ & 0xffff), (uint16_t)(lo & 0xffff), a0);
                        a1 = fma_h((uint16_t)(qa_ >> 16), (uint16_t)(lo >> 16), a1);
                        a0 = fma_h((uint16_t)(qb_ & 0xffff), (uint16_t)(hi & 0xffff), a0);
                        a1 = fma_h((uint16_t)(qb_ >> 16), (uint16_t)(hi >> 16), a1);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const uint4 kv = *reinterpret_cast<const uint4*>(st + koff[i][h]);
                        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            a0 = fma_h((uint16_t)(qh[h][e] & 0xffff), (uint16_t)(kw[e] & 0xffff), a0);
                            a1 = fma_h((uint16_t)(qh[h][e] >> 16), (uint16_t)(kw[e] >> 16), a1);
                        }
                    }
                }
                acc[i] = C::KQ ? (a0 + a1) - corr : a0 + a1;
            }
#pragma unroll
            for (int off = 1; off < 8; off <<= 1)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
            float s[4], mx = kNegInf;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                s[i] = grp + 4 * i < nv ? acc[i] * sl2 : kNegInf;
                mx = fmaxf(mx, s[i]);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mn = fmaxf(m, mx);
            const float mu = mn == kNegInf ? 0.f : mn;
            const float alpha = ex2(m - mu);
            m = mn;
            float psum = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                s[i] = ex2(s[i] - mu);
                psum += s[i];
            }
            l = l * alpha + (c == 0 ? psum : 0.f);
            if (alpha != 1.f) {
#pragma unroll
                for (int i = 0; i < DPT; ++i) o[i] *= alpha;
            }
            if (c == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) pbuf[grp + 4 * i] = __float2half_rn(s[i]);
            }
            __syncwarp();
            const uint4 pw0 = reinterpret_cast<const uint4*>(pbuf)[0];
            const uint4 pw1 = reinterpret_cast<const uint4*>(pbuf)[1];
            const uint32_t pw[8] = {pw0.x, pw0.y, pw0.z, pw0.w, pw1.x, pw1.y, pw1.z, pw1.w};
            const uint8_t* vb = st + C::V_OFF + v_byte;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                if (t < nv) {
                    const uint16_t pt = (uint16_t)(t & 1 ? pw[t >> 1] >> 16 : pw[t >> 1] & 0xffff);
                    const uint8_t* vr = vb + tile_chunk<C>(qw * 16 + t, v_cg);
                    if constexpr (DPT == 4) {
                        const uint2 vv = *reinterpret_cast<const uint2*>(vr);
                        o[0] = fma_h(pt, (uint16_t)(vv.x & 0xffff), o[0]);
                        o[1] = fma_h(pt, (uint16_t)(vv.x >> 16), o[1]);
                        o[2] = fma_h(pt, (uint16_t)(vv.y & 0xffff), o[2]);
                        o[3] = fma_h(pt, (uint16_t)(vv.y >> 16), o[3]);
                    } else {
                        const uint32_t vv = *reinterpret_cast<const uint32_t*>(vr);
                        o[0] = fma_h(pt, (uint16_t)(vv & 0xffff), o[0]);
                        o[1] = fma_h(pt, (uint16_t)(vv >> 16), o[1]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + stage * 8);

        if (md.flags & F_LAST) {
            const int tid = threadIdx.x;
            float lr = l;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) lr += __shfl_xor_sync(0xffffffffu, lr, off);
            if (lane == 0) {
                mlb[(qw * C::RP) * 2] = m;
                mlb[(qw * C::RP) * 2 + 1] = lr;
            }
            named_bar_sync(1, C::NCW * 32);
            const float f = row_factor<C>(mlb, 0, m);
            float* slice = obuf + (qw & 1) * C::OBUF_SLICE;
            for (int round = 0; round < C::TW / 2; ++round) {  // fixed order: deterministic sums
                if ((qw >> 1) == round) {
#pragma unroll
                    for (int i = 0; i < DPT; ++i)
                        slice[v_col + i] = (round ? slice[v_col + i] : 0.f) + o[i] * f;
                }
                named_bar_sync(1, C::NCW * 32);
            }
            store_segment<C>(p, md, obuf, mlb, tid);
            named_bar_sync(1, C::NCW * 32);
        }
        if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
        }
    }
}

// ---------------------------------------------------------------------------
// Tensor-core consumer for more than 16 rows per KV head (verify windows):
// each of the token warps covers every m16 row tile for its 16 tokens,
// so K and V fragments are loaded once and reused by all row tiles.  The
// query fragments are re-read each stage (conflict-free ldmatrix) from a
// per-CTA copy of the segment's query rows, which keeps registers for the
// MT output tiles.
template <class C>
__device__ void consumer_mma_mt(const Params& p, uint8_t* smem, volatile int* abort_flag)
{
    constexpr int MT = C::MT;
    const int qw = threadIdx.x >> 5;  // token warp 0..3
    const int lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t sbase = smem_u32(smem);
    const StageMeta* smeta = reinterpret_cast<const StageMeta*>(smem + C::META_OFF);
    const uint32_t full0 = sbase + C::BAR_OFF;
    const uint32_t empty0 = full0 + C::STAGES * 8;
    const uint32_t zero_row = sbase + C::ZERO_OFF;
    float* mlb = reinterpret_cast<float*>(smem + C::ML_OFF);
    float* obuf = reinterpret_cast<float*>(smem + C::OBUF_OFF);
    const float sl2 = p.scale_log2;

    const int k_tok = qw * 16 + (lane >> 4) * 8 + (lane & 7);
    const int k_sel = (lane >> 3) & 1;
    const int v_i = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int v_tok = qw * 16 + v_i;
    const int v_sel = lane >> 4;
    // this lane's ldmatrix row address in the CTA copy of the query rows
    const uint32_t qrow0 = sbase + C::QP_OFF + ((lane & 7) + ((lane >> 3) & 1) * 8) * C::QROW;

    float O[MT][C::D / 8][4];
    float m[MT][2], l[MT][2];
    float corr[MT][2];  // int8 keys: bias * row sum of q
    int lim[MT][2];

    int stage = 0;
    uint32_t phase = 0;
    for (;;) {
        if (!mbar_wait_bounded(full0 + stage * 8, phase, kWaitLimitNs)) {
            *abort_flag = 1;
            break;
        }
        const StageMeta md = smeta[stage];
        if (md.flags & F_END) break;
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        if (md.flags & F_FIRST) {
            // copy the segment's query rows out of the stage (it will be reused)
            const uint4* src = reinterpret_cast<const uint4*>(smem + stage * C::STAGE_BYTES + C::Q_OFF);
            uint4* dst = reinterpret_cast<uint4*>(smem + C::QP_OFF);
            if constexpr (!C::KQ) {
                for (int i = threadIdx.x; i < C::RP * C::QROW / 16; i += C::NCW * 32) dst[i] = src[i];
            } else {
                // int8 keys: q times the channel scales, each 16-dim chunk
                // stored in the permuted order of k8_frag (dims 0,1,4,5,8,9,12,13
                // then 2,3,6,7,10,11,14,15), so ldmatrix yields matching fragments
                constexpr int CPR = C::QROW / 16;  // 16-byte chunks per row
                const float* sc = reinterpret_cast<const float*>(smem + stage * C::STAGE_BYTES + C::SC_OFF);
                for (int i = threadIdx.x; i < C::RP * (C::D / 16); i += C::NCW * 32) {
                    const int row = i / (C::D / 16), ks = i % (C::D / 16);
                    const uint4 a = src[row * CPR + 2 * ks], b = src[row * CPR + 2 * ks + 1];
                    const float* s16 = sc + 16 * ks;
                    const uint32_t pr[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                    uint32_t q2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        q2[e] = scale_h2(pr[e], *reinterpret_cast<const float2*>(s16 + 2 * e));
                    dst[row * CPR + 2 * ks] = make_uint4(q2[0], q2[2], q2[4], q2[6]);
                    dst[row * CPR + 2 * ks + 1] = make_uint4(q2[1], q2[3], q2[5], q2[7]);
                }
            }
            named_bar_sync(2, C::NCW * 32);
            if constexpr (C::KQ) {
                // bias corrections of this lane's rows: sums of their q entries
                // (lane tig adds 32 of the 128 dims)
#pragma unroll
                for (int t = 0; t < MT; ++t)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const uint32_t* qr = reinterpret_cast<const uint32_t*>(
                            smem + C::QP_OFF + (t * 16 + gid + rr * 8) * C::QROW) + tig * 16;
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc += h2_sum(qr[e]);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                        corr[t][rr] = kCodeBias * acc;
                    }
            }
#pragma unroll
            for (int t = 0; t < MT; ++t) {
#pragma unroll
                for (int n = 0; n < C::D / 8; ++n) O[t][n][0] = O[t][n][1] = O[t][n][2] = O[t][n][3] = 0.f;
                m[t][0] = m[t][1] = kNegInf;
                l[t][0] = l[t][1] = 0.f;
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int R = t * 16 + gid + rr * 8;
                    lim[t][rr] = R < p.rows ? md.L - p.q_len + R / p.G + 1 : md.L;
                }
            }
        }
        const int nv = md.ntok - qw * 16;
        if (nv > 0) {
            float S[MT][2][4];
#pragma unroll
            for (int t = 0; t < MT; ++t)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) S[t][nt][0] = S[t][nt][1] = S[t][nt][2] = S[t][nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < C::D / 16; ++ks) {
                uint32_t b0, b1, b2, b3;
                if constexpr (C::KQ)
                    k8_frag<C>(st, qw * 16 + gid, ks, tig, b0, b1, b2, b3);
                else
                    ldsm_x4(st + tile_chunk<C>(k_tok, 2 * ks + k_sel), b0, b1, b2, b3);
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    uint32_t a[4];
                    ldsm_x4(qrow0 + t * 16 * C::QROW + ((2 * ks + (lane >> 4)) << 4), a[0], a[1], a[2],
                            a[3]);
                    mma_16816(S[t][0], a, b0, b1);
                    mma_16816(S[t][1], a, b2, b3);
                }
            }
            const int pos0 = md.t0 + qw * 16 + tig * 2;
            const int st_end = md.t0 + md.ntok;
            uint32_t pa[MT][4];
            bool rescale = false;
            float alpha[MT][2];
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                const int lim0 = min(lim[t][0], st_end), lim1 = min(lim[t][1], st_end);
                float mx[2] = {kNegInf, kNegInf};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int pos = pos0 + nt * 8 + (c & 1);
                        const float raw = C::KQ ? S[t][nt][c] - corr[t][c >> 1] : S[t][nt][c];
                        const float v = pos < ((c >> 1) ? lim1 : lim0) ? raw * sl2 : kNegInf;
                        S[t][nt][c] = v;
                        mx[c >> 1] = fmaxf(mx[c >> 1], v);
                    }
                float mu[2];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
                    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
                    const float mn = fmaxf(m[t][rr], mx[rr]);
                    mu[rr] = mn == kNegInf ? 0.f : mn;
                    alpha[t][rr] = ex2(m[t][rr] - mu[rr]);
                    m[t][rr] = mn;
                    rescale |= alpha[t][rr] != 1.f;
                }
                float ps[2] = {0.f, 0.f};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float e = ex2(S[t][nt][c] - mu[c >> 1]);
                        S[t][nt][c] = e;
                        ps[c >> 1] += e;
                    }
                l[t][0] = l[t][0] * alpha[t][0] + ps[0];
                l[t][1] = l[t][1] * alpha[t][1] + ps[1];
                pa[t][0] = pack_half2(S[t][0][0], S[t][0][1]);
                pa[t][1] = pack_half2(S[t][0][2], S[t][0][3]);
                pa[t][2] = pack_half2(S[t][1][0], S[t][1][1]);
                pa[t][3] = pack_half2(S[t][1][2], S[t][1][3]);
            }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int t = 0; t < MT; ++t)
#pragma unroll
                    for (int n = 0; n < C::D / 8; ++n) {
                        O[t][n][0] *= alpha[t][0];
                        O[t][n][1] *= alpha[t][0];
                        O[t][n][2] *= alpha[t][1];
                        O[t][n][3] *= alpha[t][1];
                    }
            }
            const bool v_ok = v_i < nv;
#pragma unroll
            for (int np = 0; np < C::D / 16; ++np) {
                const uint32_t addr =
                    v_ok ? st + C::V_OFF + tile_chunk<C>(v_tok, 2 * np + v_sel) : zero_row;
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(addr, b0, b1, b2, b3);
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    mma_16816(O[t][2 * np], pa[t], b0, b1);
                    mma_16816(O[t][2 * np + 1], pa[t], b2, b3);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + stage * 8);

        if (md.flags & F_LAST) {
            const int tid = threadIdx.x;
#pragma unroll
            for (int t = 0; t < MT; ++t)
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    float lr = l[t][rr];
                    lr += __shfl_xor_sync(0xffffffffu, lr, 1);
                    lr += __shfl_xor_sync(0xffffffffu, lr, 2);
                    if (tig == 0) {
                        const int R = t * 16 + gid + rr * 8;
                        mlb[(qw * C::RP + R) * 2] = m[t][rr];
                        mlb[(qw * C::RP + R) * 2 + 1] = lr;
                    }
                }
            named_bar_sync(1, C::NCW * 32);
            float* slice = obuf + (qw & 1) * C::OBUF_SLICE;
            for (int round = 0; round < C::TW / 2; ++round) {
                if ((qw >> 1) == round) {
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        const int R0 = t * 16 + gid, R1 = R0 + 8;
                        const bool row0 = R0 < p.rows, row1 = R1 < p.rows;
                        const float f0 = row0 ? row_factor<C>(mlb, R0, m[t][0]) : 0.f;
                        const float f1 = row1 ? row_factor<C>(mlb, R1, m[t][1]) : 0.f;
                        float* r0p = slice + R0 * C::OB_STRIDE + tig * 2;
                        float* r1p = slice + R1 * C::OB_STRIDE + tig * 2;
                        float2 x0[C::D / 8], x1[C::D / 8];  // loads first, then stores
#pragma unroll
                        for (int n = 0; n < C::D / 8; ++n) {
                            x0[n] = make_float2(0.f, 0.f);
                            x1[n] = make_float2(0.f, 0.f);
                            if (round && row0) x0[n] = *reinterpret_cast<const float2*>(r0p + n * 8);
                            if (round && row1) x1[n] = *reinterpret_cast<const float2*>(r1p + n * 8);
                        }
#pragma unroll
                        for (int n = 0; n < C::D / 8; ++n) {
                            if (row0)
                                *reinterpret_cast<float2*>(r0p + n * 8) =
                                    make_float2(x0[n].x + O[t][n][0] * f0, x0[n].y + O[t][n][1] * f0);
                            if (row1)
                                *reinterpret_cast<float2*>(r1p + n * 8) =
                                    make_float2(x1[n].x + O[t][n][2] * f1, x1[n].y + O[t][n][3] * f1);
                        }
                    }
                }
                named_bar_sync(1, C::NCW * 32);
            }
            store_segment<C>(p, md, obuf, mlb, tid);
            named_bar_sync(1, C::NCW * 32);
        }
        if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
        }
    }
}

// ---------------------------------------------------------------------------
// Tensor-core consumer with the tokens as the MMA's M dimension: per warp and
// stage, S^T (16 tokens x 8*NR8 rows) = K Q^T and O^T (head dims x rows) +=
// V^T P^T, mma.sync m16n8k16.  No row padding to 16 (a GQA group of 8 fills
// one n8 tile), half the MMAs and half the accumulator registers of the
// rows-as-M form.  P^T reaches the B-operand layout of the P V product with
// movmatrix (an 8x8 transpose in registers).  Each thread owns rows 2*tig,
// 2*tig+1 of every row tile for two tokens (gid, gid + 8): a row's softmax
// maximum and sum reduce over the 8 lanes of one tig.
template <class C>
__device__ void consumer_tc(const Params& p, uint8_t* smem, volatile int* abort_flag)
{
    constexpr int NR = C::NR8;
    constexpr int KS = C::D / 16;
    const int qw = threadIdx.x >> 5;  // token warp
    const int lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t sbase = smem_u32(smem);
    const StageMeta* smeta = reinterpret_cast<const StageMeta*>(smem + C::META_OFF);
    const uint32_t full0 = sbase + C::BAR_OFF;
    const uint32_t empty0 = full0 + C::STAGES * 8;
    const uint32_t zero_row = sbase + C::ZERO_OFF;
    float* mlb = reinterpret_cast<float*>(smem + C::ML_OFF);
    const float sl2 = p.scale_log2;

    // ldmatrix lane geometry.  K as the A operand: matrices (tokens 0-7 |
    // 8-15) x (dims lo | hi); V^T as the A operand (transposed load):
    // matrices (dims lo | hi) x (tokens 0-7 | 8-15); query rows as the B
    // operand: row lane & 7 of a row tile, 16-byte chunk lane >> 3.
    const int a_i = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int a_sel = lane >> 4;
    const int v_i = (lane >> 4) * 8 + (lane & 7);
    const int v_sel = (lane >> 3) & 1;

    float O[KS][NR][4];  // O^T tile (dims 16*np.., rows 8*nt..): d = gid(+8), r = 2tig(+1)
    uint32_t qb[C::QPERSIST ? 1 : KS][NR][2];  // B fragments of the query rows
    float m[NR][2], l[NR][2];
    float corr[NR][2];  // int8 keys: bias * row sum of the scaled q, in log2 units (x scale)
    int lim[NR][2];

    // B fragments of k-steps ks, ks+1 of row tile nt from padded query rows at `rows`
    auto load_qb2 = [&](uint32_t rows, int nt, int ks, uint32_t (&b)[4]) {
        ldsm_x4(rows + (nt * 8 + (lane & 7)) * C::QROW + ((2 * ks + (lane >> 3)) << 4), b[0], b[1],
                b[2], b[3]);
    };

    int stage = 0;
    uint32_t phase = 0;
    for (;;) {
        if (!mbar_wait_bounded(full0 + stage * 8, phase, kWaitLimitNs)) {
            *abort_flag = 1;
            break;
        }
        const StageMeta md = smeta[stage];
        if (md.flags & F_END) break;
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        if (md.flags & F_FIRST) {
            uint32_t qsrc = st + C::Q_OFF;
            if constexpr (C::QPERSIST) {
                // copy the segment's query rows out of the stage (read every stage)
                const uint4* src = reinterpret_cast<const uint4*>(smem + stage * C::STAGE_BYTES + C::Q_OFF);
                uint4* dst = reinterpret_cast<uint4*>(smem + C::QP_OFF);
                constexpr int CPR = C::QROW / 16;  // 16-byte chunks per padded row
                if constexpr (!C::KQ) {
                    for (int i = threadIdx.x; i < C::RP * CPR; i += C::NCW * 32) dst[i] = src[i];
                } else {
                    // q times the channel scales, each 16-dim chunk stored in the
                    // permuted order of the int8 key fragments (dims 0,1,4,5,8,9,
                    // 12,13 then 2,3,6,7,10,11,14,15)
                    const float* sc = reinterpret_cast<const float*>(smem + stage * C::STAGE_BYTES + C::SC_OFF);
                    for (int i = threadIdx.x; i < C::RP * KS; i += C::NCW * 32) {
                        const int row = i / KS, ks = i % KS;
                        const uint4 a = src[row * CPR + 2 * ks], b = src[row * CPR + 2 * ks + 1];
                        const float* s16 = sc + 16 * ks;
                        const uint32_t pr[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                        uint32_t q2[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            q2[e] = scale_h2(pr[e], *reinterpret_cast<const float2*>(s16 + 2 * e));
                        dst[row * CPR + 2 * ks] = make_uint4(q2[0], q2[2], q2[4], q2[6]);
                        dst[row * CPR + 2 * ks + 1] = make_uint4(q2[1], q2[3], q2[5], q2[7]);
                    }
                }
                named_bar_sync(2, C::NCW * 32);
                qsrc = sbase + C::QP_OFF;
            } else if constexpr (!C::KQ) {
#pragma unroll
                for (int nt = 0; nt < NR; ++nt)
#pragma unroll
                    for (int ks = 0; ks < KS; ks += 2) {
                        uint32_t b[4];
                        load_qb2(qsrc, nt, ks, b);
                        qb[ks][nt][0] = b[0];
                        qb[ks][nt][1] = b[1];
                        qb[ks + 1][nt][0] = b[2];
                        qb[ks + 1][nt][1] = b[3];
                    }
            } else {
                // int8 keys: q of row nt*8+gid times the channel scales, in the
                // permuted dim order (lane tig: dims 4tig, 4tig+1 | 4tig+2, 4tig+3)
                const float* sc = reinterpret_cast<const float*>(smem + stage * C::STAGE_BYTES + C::SC_OFF);
#pragma unroll
                for (int nt = 0; nt < NR; ++nt) {
                    const uint8_t* qr = smem + stage * C::STAGE_BYTES + C::Q_OFF + (nt * 8 + gid) * C::QROW;
                    const float* sch = sc + (C::HP > 1 ? nt * C::D : 0);  // row tile nt's head
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const int d = 16 * ks + 4 * tig;
                        qb[ks][nt][0] = scale_h2(*reinterpret_cast<const uint32_t*>(qr + d * 2),
                                                 *reinterpret_cast<const float2*>(sch + d));
                        qb[ks][nt][1] = scale_h2(*reinterpret_cast<const uint32_t*>(qr + d * 2 + 4),
                                                 *reinterpret_cast<const float2*>(sch + d + 2));
                    }
                }
            }
            if constexpr (C::KQ) {
                // bias corrections of this thread's rows 8nt + 2tig (+1): sums of
                // their scaled q entries (lane tig adds 32 of the 128 dims of row
                // 8nt + gid, then the row sums are fetched from lane 4*row)
#pragma unroll
                for (int nt = 0; nt < NR; ++nt) {
                    float acc = 0.f;
                    if constexpr (C::QPERSIST) {
                        const uint32_t* qr = reinterpret_cast<const uint32_t*>(
                            smem + C::QP_OFF + (nt * 8 + gid) * C::QROW) + tig * 16;
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc += h2_sum(qr[e]);
                    } else {
#pragma unroll
                        for (int ks = 0; ks < KS; ++ks) acc += h2_sum(qb[ks][nt][0]) + h2_sum(qb[ks][nt][1]);
                    }
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                    corr[nt][0] = kCodeBias * sl2 * __shfl_sync(0xffffffffu, acc, (2 * tig) * 4);
                    corr[nt][1] = kCodeBias * sl2 * __shfl_sync(0xffffffffu, acc, (2 * tig + 1) * 4);
                }
            }
#pragma unroll
            for (int np = 0; np < KS; ++np)
#pragma unroll
                for (int nt = 0; nt < NR; ++nt) O[np][nt][0] = O[np][nt][1] = O[np][nt][2] = O[np][nt][3] = 0.f;
#pragma unroll
            for (int nt = 0; nt < NR; ++nt)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int R = nt * 8 + 2 * tig + i;
                    m[nt][i] = kNegInf;
                    l[nt][i] = 0.f;
                    int j = 0;
                    lim[nt][i] = row_head(p, md.kvh, R, j) >= 0 ? md.L - p.q_len + j + 1 : md.L;
                }
        }
#pragma unroll 1
        for (int sub = 0; sub < C::SUBS; ++sub) {
        const int tb = (qw * C::SUBS + sub) * 16;  // first stage token of this sub-tile
        const int nv = md.ntok - tb;
        if (nv > 0) {
            const int a_tok = tb + a_i, v_tok = tb + v_i;
            // S^T = K Q^T for my 16 tokens; the k-steps accumulate into NCH
            // separate chains (fewer dependent MMAs in a row), summed after
            constexpr int NCH = NR == 1 ? 4 : 2;
            float Sc[NCH][NR][4];
#pragma unroll
            for (int c = 0; c < NCH; ++c)
#pragma unroll
                for (int nt = 0; nt < NR; ++nt) Sc[c][nt][0] = Sc[c][nt][1] = Sc[c][nt][2] = Sc[c][nt][3] = 0.f;
            const uint32_t qrows = sbase + C::QP_OFF;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                float (&S)[NR][4] = Sc[ks % NCH];
                if constexpr (C::HP > 1) {
                    // row tile nt is head nt of the pair: its own K rows
#pragma unroll
                    for (int nt = 0; nt < NR; ++nt) {
                        uint32_t a[4];
                        if constexpr (C::KQ) {
                            i8x4_to_h2x2_biased(lds_u32(st + tile_chunk_k8<C>(tb + gid, ks, nt) + 4 * tig), a[0],
                                                a[2]);
                            i8x4_to_h2x2_biased(lds_u32(st + tile_chunk_k8<C>(tb + gid + 8, ks, nt) + 4 * tig),
                                                a[1], a[3]);
                        } else {
                            ldsm_x4(st + tile_chunk<C>(a_tok, 2 * ks + a_sel, nt), a[0], a[1], a[2], a[3]);
                        }
                        mma_16816(S[nt], a, qb[ks][nt][0], qb[ks][nt][1]);
                    }
                    continue;
                }
                uint32_t a[4];
                if constexpr (C::KQ) {
                    // tokens gid and gid + 8, dims 16ks + 4tig .. +3 (permuted order)
                    i8x4_to_h2x2_biased(lds_u32(st + tile_chunk_k8<C>(tb + gid, ks) + 4 * tig), a[0], a[2]);
                    i8x4_to_h2x2_biased(lds_u32(st + tile_chunk_k8<C>(tb + gid + 8, ks) + 4 * tig), a[1], a[3]);
                } else {
                    ldsm_x4(st + tile_chunk<C>(a_tok, 2 * ks + a_sel), a[0], a[1], a[2], a[3]);
                }
                if constexpr (C::QPERSIST) {
#pragma unroll
                    for (int nt = 0; nt < NR; nt += 2) {
                        // two row tiles per load: (tile nt | nt+1) x (chunk 2ks | 2ks+1)
                        uint32_t b[4];
                        const int row = nt * 8 + (lane & 7) + ((lane >> 4) & 1) * 8;
                        ldsm_x4(qrows + row * C::QROW + ((2 * ks + ((lane >> 3) & 1)) << 4), b[0], b[1], b[2],
                                b[3]);
                        mma_16816(S[nt], a, b[0], b[1]);
                        if (nt + 1 < NR) mma_16816(S[nt + 1], a, b[2], b[3]);
                    }
                } else {
#pragma unroll
                    for (int nt = 0; nt < NR; ++nt) mma_16816(S[nt], a, qb[ks][nt][0], qb[ks][nt][1]);
                }
            }
            float S[NR][4];
#pragma unroll
            for (int nt = 0; nt < NR; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v = Sc[0][nt][e];
#pragma unroll
                    for (int c = 1; c < NCH; ++c) v += Sc[c][nt][e];
                    S[nt][e] = v;
                }
            // mask: a token counts if the row may see it and this stage loaded
            // it; a sub-tile that every row sees whole (the usual case) skips it
            const int pos0 = md.t0 + tb + gid;
            const int st_end = md.t0 + md.ntok;
            const bool whole = md.t0 + tb + 16 <= min(md.L - p.q_len + 1, st_end);
            // Each row keeps a reference maximum m shared by the 8 lanes that
            // hold its tokens; it is raised (a shuffle reduction, O rescaled)
            // only when some score of the sub-tile passes it by more than
            // 2^kRescaleThreshold, so most sub-tiles cost one vote and the
            // weights stay below 2^kRescaleThreshold (exact after the final
            // division by l, which uses the same reference).  Scores stay raw
            // dot products (over int8 keys: biased); the score in log2 units,
            // raw * sl2 - corr (corr: the int8 bias in log2 units), is formed
            // inside each exponential's argument by one FMA.
            bool rescale = false;
            float alpha[NR][2], mu[NR][2], mx[NR][2];
            bool over = false;
#pragma unroll
            for (int nt = 0; nt < NR; ++nt) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (!whole) {
                        const int lm = min(lim[nt][i], st_end);
                        S[nt][i] = pos0 < lm ? S[nt][i] : kNegInf;
                        S[nt][2 + i] = pos0 + 8 < lm ? S[nt][2 + i] : kNegInf;
                    }
                    mx[nt][i] = fmaf(fmaxf(S[nt][i], S[nt][2 + i]), sl2, C::KQ ? -corr[nt][i] : 0.f);
                    over |= mx[nt][i] > m[nt][i] + kRescaleThreshold;
                    alpha[nt][i] = 1.f;
                    mu[nt][i] = m[nt][i] == kNegInf ? 0.f : m[nt][i];
                }
            }
            if (__any_sync(0xffffffffu, over)) {
#pragma unroll
                for (int nt = 0; nt < NR; ++nt) {
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1)
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            mx[nt][i] = fmaxf(mx[nt][i], __shfl_xor_sync(0xffffffffu, mx[nt][i], off));
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float mn = fmaxf(m[nt][i], mx[nt][i]);
                        mu[nt][i] = mn == kNegInf ? 0.f : mn;
                        alpha[nt][i] = ex2(m[nt][i] - mu[nt][i]);
                        m[nt][i] = mn;
                        rescale |= alpha[nt][i] != 1.f;
                    }
                }
            }
            uint32_t pb[NR][2];
#pragma unroll
            for (int nt = 0; nt < NR; ++nt) {
                const float b0 = C::KQ ? mu[nt][0] + corr[nt][0] : mu[nt][0];
                const float b1 = C::KQ ? mu[nt][1] + corr[nt][1] : mu[nt][1];
                const float e0 = ex2(fmaf(S[nt][0], sl2, -b0)), e1 = ex2(fmaf(S[nt][1], sl2, -b1));
                const float e2 = ex2(fmaf(S[nt][2], sl2, -b0)), e3 = ex2(fmaf(S[nt][3], sl2, -b1));
                l[nt][0] = l[nt][0] * alpha[nt][0] + (e0 + e2);
                l[nt][1] = l[nt][1] * alpha[nt][1] + (e1 + e3);
                // P^T (tokens x rows) -> P (rows x tokens) fragments: b0 = P[gid][2tig..],
                // b1 = P[gid][8 + 2tig..]
                pb[nt][0] = movmatrix_trans(pack_half2(e0, e1));
                pb[nt][1] = movmatrix_trans(pack_half2(e2, e3));
            }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int np = 0; np < KS; ++np)
#pragma unroll
                    for (int nt = 0; nt < NR; ++nt) {
                        O[np][nt][0] *= alpha[nt][0];
                        O[np][nt][1] *= alpha[nt][1];
                        O[np][nt][2] *= alpha[nt][0];
                        O[np][nt][3] *= alpha[nt][1];
                    }
            }
            // O^T += V^T P^T; rows of V past the valid tokens read a zero row
            const bool v_ok = v_i < nv;
#pragma unroll
            for (int np = 0; np < KS; ++np) {
                if constexpr (C::HP > 1) {
#pragma unroll
                    for (int nt = 0; nt < NR; ++nt) {  // head nt's V rows
                        const uint32_t addr =
                            v_ok ? st + C::V_OFF + tile_chunk<C>(v_tok, 2 * np + v_sel, nt) : zero_row;
                        uint32_t a[4];
                        ldsm_x4_trans(addr, a[0], a[1], a[2], a[3]);
                        mma_16816(O[np][nt], a, pb[nt][0], pb[nt][1]);
                    }
                } else {
                    const uint32_t addr = v_ok ? st + C::V_OFF + tile_chunk<C>(v_tok, 2 * np + v_sel) : zero_row;
                    uint32_t a[4];
                    ldsm_x4_trans(addr, a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NR; ++nt) mma_16816(O[np][nt], a, pb[nt][0], pb[nt][1]);
                }
            }
        }
        }
        __syncwarp();
        if (!(md.flags & F_LAST)) {
            if (lane == 0) mbar_arrive(empty0 + stage * 8);
        } else {
            // Segment end: merge the token-warps.  The stage just consumed is
            // kept (not yet released) and its shared memory holds one slice per
            // warp: each warp writes its o scaled by 2^(m_w - M) / L, then one
            // pass sums the slices in warp order and stores.
            const int tid = threadIdx.x;
#pragma unroll
            for (int nt = 0; nt < NR; ++nt)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float lr = l[nt][i];
                    lr += __shfl_xor_sync(0xffffffffu, lr, 4);
                    lr += __shfl_xor_sync(0xffffffffu, lr, 8);
                    lr += __shfl_xor_sync(0xffffffffu, lr, 16);
                    if (gid == 0) {
                        const int R = nt * 8 + 2 * tig + i;
                        mlb[(qw * C::RP + R) * 2] = m[nt][i];
                        mlb[(qw * C::RP + R) * 2 + 1] = lr;
                    }
                }
            named_bar_sync(1, C::NCW * 32);  // every warp done with the stage's tiles
            float* slices = reinterpret_cast<float*>(smem + stage * C::STAGE_BYTES);
            // this warp's o times its factor into slot qw mod MSLOTS: written by
            // the upper warps first, then added to by the lower ones (a fixed
            // order: bit-reproducible)
            auto put = [&](bool add) {
#pragma unroll
                for (int nt = 0; nt < NR; ++nt) {
                    const float f0 = row_factor<C>(mlb, nt * 8 + 2 * tig, m[nt][0]);
                    const float f1 = row_factor<C>(mlb, nt * 8 + 2 * tig + 1, m[nt][1]);
                    float* r0 = slices + ((qw % C::MSLOTS) * C::RP + nt * 8 + 2 * tig) * C::OB_STRIDE + gid;
                    float* r1 = r0 + C::OB_STRIDE;
#pragma unroll
                    for (int np = 0; np < KS; ++np) {
                        r0[16 * np] = (add ? r0[16 * np] : 0.f) + O[np][nt][0] * f0;
                        r1[16 * np] = (add ? r1[16 * np] : 0.f) + O[np][nt][1] * f1;
                        r0[16 * np + 8] = (add ? r0[16 * np + 8] : 0.f) + O[np][nt][2] * f0;
                        r1[16 * np + 8] = (add ? r1[16 * np + 8] : 0.f) + O[np][nt][3] * f1;
                    }
                }
            };
            if constexpr (C::MSLOTS == C::TW) {
                put(false);
            } else {
                if (qw >= C::MSLOTS) put(false);
                named_bar_sync(1, C::NCW * 32);
                if (qw < C::MSLOTS) put(true);
            }
            named_bar_sync(1, C::NCW * 32);
            store_segment_slices<C>(p, md, slices, mlb, tid);
            // the slices and mlb are read: the stage may be refilled (by the
            // async proxy, after these generic accesses) and mlb rewritten
            fence_proxy_async();
            named_bar_sync(1, C::NCW * 32);
            if (lane == 0) mbar_arrive(empty0 + stage * 8);
        }
        if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
        }
    }
}

// ---------------------------------------------------------------------------
// tcgen05 consumer (query rows > 1, head_dim 128): both products on the
// 5th-generation tensor cores, accumulators in tensor memory.
//
// Each 128-token stage is one MMA pair over all 128 TMEM lanes.  Lane m holds
// query row r = m mod R (R = UMR, the padded rows) and owns the stage's
// tokens [g*R, g*R + R), g = m / R: the rows are replicated 128/R times so
// that every lane, and so every softmax thread, has work.
//   S = Q K^T   M128 N128 K128, A = the replicated query rows (fp16 pairs in
//               tensor memory), B = the stage's K (K-major, 128-byte swizzle)
//   softmax     thread m = lane m: its R scores, its own running maximum and
//               denominator (online softmax over its tokens only; no
//               cross-thread reduction per stage)
//   O += P V    M128 N128 K128, A = P (fp16 pairs in tensor memory, zero
//               outside the lane's tokens), B = the stage's V (MN-major)
// At a segment's end the 128/R partial (o, m, l) of each row are combined in
// a fixed order (bit-reproducible) through the consumed stage's shared
// memory.  The MMAs do 128/R times the useful flops; at 128 tokens per stage
// that is ~1000 tensor cycles against ~2700 of HBM time per stage.
// Int8 keys: the softmax warps widen the stage's codes to fp16 in place (the
// channel scales are folded into the query rows).
// Tensor memory: S (128 columns), P (two buffers of 64), O (128), the query
// rows (two buffers of 64, by segment parity).
enum : uint32_t { UM_S = 0, UM_P = 128, UM_O = 256, UM_Q = 384, UM_COLS = 512 };
enum : int { UB_S_FULL = 0, UB_S_FREE = 1, UB_P_FULL = 2, UB_O_DONE = 4, UB_Q_READY = 6, UB_KDQ = 7,
             UB_EP = 8, UB_DRAIN = 9 };

template <class C>
__device__ void consumer_um(const Params& p, uint8_t* smem, uint32_t tmem, volatile int* abort_flag)
{
    constexpr int R = C::UMR;        // padded rows; also tokens per lane (128 tokens / (128 / R) lanes)
    constexpr int T = R;
    constexpr int NG = 128 / R;      // lanes per query row
    constexpr int NSUB = 32 / T;     // token groups in a warp's 32 tokens
    constexpr int HW = T / 2;        // fp16 pairs of a lane's weights
    static_assert(C::TS == 128 && C::NCW == 4, "one 128-lane MMA per stage");
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m = threadIdx.x;       // TMEM lane
    const int r = m % R;
    const int sub = lane / T;
    const uint32_t sbase = smem_u32(smem);
    const StageMeta* smeta = reinterpret_cast<const StageMeta*>(smem + C::META_OFF);
    const uint32_t full0 = sbase + C::BAR_OFF;
    const uint32_t empty0 = full0 + C::STAGES * 8;
    const uint32_t ub = sbase + C::UB_OFF;
    const uint32_t lb = tmem + ((uint32_t)(32 * w) << 16);  // this warp's lane quarter
    float* ml = reinterpret_cast<float*>(smem + C::ML_OFF);
    const float sl2 = p.scale_log2;
    const bool row_ok = r < p.rows;
    const int jr = row_ok ? r / p.G : 0;

    {   // both weight buffers start zero; each warp only ever writes its own tokens' columns
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
#pragma unroll
        for (int c = 0; c < 128; c += 32) tmem_st32(lb + UM_P + c, z);
        tmem_wait_st();
    }

    bool ok = true;
    // every lane waits; the warp stops together when any lane gave up.  A
    // loader that gave up still posts the end marker, so the compute warps
    // stop there, all at the same stage (they do not read the abort flag:
    // one warp stopping early would leave the others at the merge barrier)
    auto wait_all = [&](uint32_t bar, uint32_t par) -> bool {
        const bool got = mbar_wait_bounded(bar, par, kWaitLimitNs);
        const bool all = __all_sync(0xffffffffu, got);
        if (!all) ok = false;
        return all;
    };
    int ep = 0;  // phases of the epilogue barrier used so far
    auto ep_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(ub + 8 * UB_EP);
        const bool got = wait_all(ub + 8 * UB_EP, (uint32_t)(ep & 1));
        ++ep;
        return got;
    };

    // Everything stage `st` needs before its S can be issued, done by each
    // warp for its lanes / tokens: the segment's query rows into tensor
    // memory (first stage of a segment; the buffers alternate by segment),
    // int8 codes widened to fp16, V rows past the staged tokens zeroed.
    int qseg = 0;  // segments whose query rows are written
    auto prep = [&](int st, const StageMeta& mdd) {
        uint8_t* sg = smem + st * C::STAGE_BYTES;
        if (mdd.flags & F_FIRST) {
            // row r in lane m (times the channel scales over int8 keys);
            // padded rows are zero
            const uint4* qs = reinterpret_cast<const uint4*>(sg + C::Q_OFF + r * C::QROW);
            const uint32_t qcol = UM_Q + (uint32_t)((qseg & 1) * 64);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float qv[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 x = qs[h * 8 + i];
                    uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if constexpr (C::KQ) {
                            const float* sc = reinterpret_cast<const float*>(sg + C::SC_OFF);
                            const int d = 2 * (h * 32 + i * 4 + e);
                            wv[e] = scale_h2(wv[e], *reinterpret_cast<const float2*>(sc + d));
                        }
                        qv[i * 4 + e] = __uint_as_float(wv[e]);
                    }
                }
                tmem_st32(lb + qcol + 32 * h, qv);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ub + 8 * UB_Q_READY);
            ++qseg;
        }
        if constexpr (C::KQ) {
            // token m's 128 codes (swizzled 16-byte chunks in the upper half of
            // K) -> fp16 in both halves; the thread reads its whole row first,
            // so the in-place widening never races another thread
            const uint32_t kb = smem_u32(sg);
            uint4 cw[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                cw[c] = *reinterpret_cast<const uint4*>(sg + C::UM_HALF + m * 128 + ((c ^ (m & 7)) << 4));
            const uint32_t bias = 0x64806480u;  // fp16 pair (1152, 1152)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t cwords[4] = {cw[c].x, cw[c].y, cw[c].z, cw[c].w};
                uint32_t hw[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    uint32_t lo, hi;
                    i8x4_to_h2x2_biased(cwords[e], lo, hi);
                    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hw[2 * e]) : "r"(lo), "r"(bias));
                    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hw[2 * e + 1]) : "r"(hi), "r"(bias));
                }
                // dims 16c .. 16c+7 and 16c+8 .. 16c+15: chunks 2c, 2c+1 of the row
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int dc = 2 * c + q;
                    const uint32_t addr = kb + (uint32_t)((dc >> 3) * C::UM_HALF + m * 128 +
                                                          (((dc & 7) ^ (m & 7)) << 4));
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(hw[4 * q]),
                                 "r"(hw[4 * q + 1]), "r"(hw[4 * q + 2]), "r"(hw[4 * q + 3])
                                 : "memory");
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(ub + 8 * UB_KDQ);
        }
        if (mdd.ntok < C::TS && m >= mdd.ntok) {
            // V rows past the staged tokens must be finite zeros for the MMA
            // (ordered before the tensor core's read by the fence ahead of
            // this stage's weights-written arrive)
            uint8_t* vr = sg + C::V_OFF + m * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                *reinterpret_cast<uint4*>(vr + (c << 4)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(vr + C::UM_HALF + (c << 4)) = make_uint4(0, 0, 0, 0);
            }
        }
    };

    float m_run = kNegInf, l_run = 0.f;
    int stage = 0, j = 0, prepped = -1;
    uint32_t phase = 0;
    for (;;) {
        if (!wait_all(full0 + stage * 8, phase)) break;
        const StageMeta md = smeta[stage];
        if (md.flags & F_END) break;
        uint8_t* stg = smem + stage * C::STAGE_BYTES;
        if (prepped != j) prep(stage, md);
        if (md.flags & F_FIRST) {
            m_run = kNegInf;
            l_run = 0.f;
        }
        // ---- scores of this stage
        if (!wait_all(ub + 8 * UB_S_FULL, (uint32_t)(j & 1))) break;
        tc_fence_after();
        float x[32];
        tmem_ld32(lb + UM_S + 32 * w, x);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ub + 8 * UB_S_FREE);
        {   // prepare the next stage now if it has landed (lane 0 decides)
            const int ns = stage + 1 == C::STAGES ? 0 : stage + 1;
            const uint32_t np = stage + 1 == C::STAGES ? phase ^ 1u : phase;
            const bool landed = __shfl_sync(0xffffffffu, mbar_test(full0 + ns * 8, np) ? 1 : 0, 0) != 0;
            if (landed) {
                const StageMeta nmd = smeta[ns];
                if (!(nmd.flags & F_END)) {
                    prep(ns, nmd);
                    prepped = j + 1;
                }
            }
        }
        float v[T];
#pragma unroll
        for (int i = 0; i < T; ++i) {
            v[i] = x[i];
#pragma unroll
            for (int s2 = 1; s2 < NSUB; ++s2)
                if (sub == s2) v[i] = x[s2 * T + i];
        }
        // visible: staged (< ntok) and, in a verify window, up to the row's position
        int lim = md.L - p.q_len + jr + 1 - md.t0;
        if (lim > md.ntok) lim = md.ntok;
        if (!row_ok) lim = 0;
        const int nvis = lim - (32 * w + sub * T);
        float mx = kNegInf;
#pragma unroll
        for (int i = 0; i < T; ++i) {
            v[i] = i < nvis ? v[i] : kNegInf;
            mx = fmaxf(mx, v[i]);
        }
        mx *= sl2;
        const bool grow = mx > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, grow)) {
            const float mn = grow ? mx : m_run;
            const float alpha = m_run == kNegInf ? 1.f : ex2(m_run - mn);
            if (__any_sync(0xffffffffu, grow && m_run != kNegInf)) {
                // O holds this segment's earlier stages: P V(j-1) (issued right
                // after S(j)) must have finished before it is rescaled
                const int jp = j - 1;
                if (!wait_all(ub + 8 * (UB_O_DONE + (jp & 1)), (uint32_t)((jp >> 1) & 1))) break;
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < C::D; c0 += 32) {
                    float o[32];
                    tmem_ld32(lb + UM_O + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(lb + UM_O + c0, o);
                }
                tmem_wait_st();
            }
            l_run *= alpha;
            m_run = mn;
        }
        const float mu = m_run == kNegInf ? 0.f : m_run;
        uint32_t pw[HW];
        float ls = 0.f;
#pragma unroll
        for (int e = 0; e < HW; ++e) {
            const float a = ex2(fmaf(v[2 * e], sl2, -mu));
            const float b = ex2(fmaf(v[2 * e + 1], sl2, -mu));
            ls += a + b;
            pw[e] = pack_half2(a, b);
        }
        l_run += ls;
        // weight buffer j&1 was last read by P V(j-2)
        if (j >= 2 && !wait_all(ub + 8 * (UB_O_DONE + (j & 1)), (uint32_t)(((j - 2) >> 1) & 1))) break;
        float pv[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pv[c] = (c / HW == sub) ? __uint_as_float(pw[c % HW]) : 0.f;
        tmem_st16(lb + UM_P + (uint32_t)((j & 1) * 64 + 16 * w), pv);
        tmem_wait_st();
        fence_proxy_async();  // the V zeros above are read by the tensor core
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ub + 8 * (UB_P_FULL + (j & 1)));

        if (md.flags & F_LAST) {
            // ---- segment end: combine the NG partials of every row
            if (!wait_all(ub + 8 * (UB_O_DONE + (j & 1)), (uint32_t)((j >> 1) & 1))) break;
            tc_fence_after();
            ml[2 * m] = m_run;
            ml[2 * m + 1] = l_run;
            if (!ep_sync()) break;
            float M = kNegInf;
#pragma unroll
            for (int g = 0; g < NG; ++g) M = fmaxf(M, ml[2 * (g * R + r)]);
            const float Mu = M == kNegInf ? 0.f : M;
            float Ls = 0.f;
#pragma unroll
            for (int g = 0; g < NG; ++g) Ls += ml[2 * (g * R + r) + 1] * ex2(ml[2 * (g * R + r)] - Mu);
            const float f = Ls > 0.f ? ex2(m_run - Mu) / Ls : 0.f;
            // lane m's o times its factor -> row m of the consumed stage's K/V
            // area (512 B per row, 16-byte chunk ch stored at ch ^ (m mod 8))
#pragma unroll
            for (int c0 = 0; c0 < C::D; c0 += 32) {
                float o[32];
                tmem_ld32(lb + UM_O + c0, o);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int ch = c0 / 4 + q;
                    *reinterpret_cast<float4*>(stg + m * 512 + ((ch ^ (m & 7)) << 4)) =
                        make_float4(o[4 * q] * f, o[4 * q + 1] * f, o[4 * q + 2] * f, o[4 * q + 3] * f);
                }
            }
            if (!ep_sync()) break;
            const bool whole = (md.flags & F_WHOLE) != 0;
            const int64_t pbase = ((int64_t)blockIdx.x * 2 + md.slot) * C::RP;
            for (int idx = m; idx < p.rows * 32; idx += 128) {
                const int rr = idx >> 5, ch = idx & 31;
                float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    const int row = g * R + rr;
                    const float4 b = *reinterpret_cast<const float4*>(stg + row * 512 + ((ch ^ (row & 7)) << 4));
                    a = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
                }
                if (whole) {
                    const int jj = rr / p.G, gg = rr % p.G;
                    __half* dst = p.out + (((int64_t)md.s * p.q_len + jj) * p.Hq + (int64_t)md.kvh * p.G + gg) *
                                              C::D + ch * 4;
                    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_half2(a.x, a.y), pack_half2(a.z, a.w));
                } else {
                    *reinterpret_cast<float4*>(p.part_o + (pbase + rr) * C::D + ch * 4) = a;
                }
            }
            if (!whole && m < p.rows) p.part_lse[pbase + m] = Ls > 0.f ? Mu + lg2(Ls) : kNegInf;
            fence_proxy_async();  // generic accesses of the stage before its next copy
            if (!ep_sync()) break;
            if (m == 0) mbar_arrive(empty0 + stage * 8);
        }
        ++j;
        if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
        }
    }
    if (!ok && lane == 0) {
        atomicOr(p.err, KV_DEV_TIMEOUT);
        *abort_flag = 1;
    }
}

// MMA-issuing warp of the tcgen05 consumer (one thread issues, polling).
// S(k) needs its stage staged (and widened, for int8 keys), the segment's
// query rows in tensor memory, and the softmax done reading S(k-1); P V(i)
// needs the weights of stage i.  Whichever is ready is issued first, P V in
// stage order, so a P V never waits behind the next stage's copy.  At a
// segment boundary every earlier P V goes before the new segment's first S
// (the softmax waits for the last one before it merges the segment).  P V(i)
// releases its stage, except at a segment end, where the softmax uses the
// stage for the merge and releases it itself.
template <class C>
__device__ void mma_um(const Params& p, uint8_t* smem, uint32_t tmem, volatile int* abort_flag)
{
    const int lane = threadIdx.x & 31;
    if (lane == 0) {
        const uint32_t sbase = smem_u32(smem);
        const StageMeta* smeta = reinterpret_cast<const StageMeta*>(smem + C::META_OFF);
        const uint32_t full0 = sbase + C::BAR_OFF;
        const uint32_t empty0 = full0 + C::STAGES * 8;
        const uint32_t ub = sbase + C::UB_OFF;
        constexpr uint32_t idS = idesc_f16(128, C::TS, false);
        constexpr uint32_t idO = idesc_f16(128, C::D, true);
        // stages whose S is issued and P V is not: ring slot and flags
        constexpr int kPend = 4;
        int pst[kPend];
        int32_t pfl[kPend];
        int k = 0, pv = 0, seg = 0, stage = 0;
        uint32_t phase = 0;
        bool have_md = false, end = false, ok = true;
        int32_t flags = 0;
        uint32_t idle = 0;
        uint64_t t_idle = 0;
        while (ok) {
            bool prog = false;
            if (pv < k && mbar_test(ub + 8 * (UB_P_FULL + (pv & 1)), (uint32_t)((pv >> 1) & 1))) {
                tc_fence_after();
                const int i = pv % kPend;
                const uint32_t vb = sbase + pst[i] * C::STAGE_BYTES + C::V_OFF;
                const uint32_t pa = tmem + UM_P + (uint32_t)((pv & 1) * 64);
                const bool first = (pfl[i] & F_FIRST) != 0;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16_ts(tmem + UM_O, pa + kk * 8, smem_desc(vb + kk * 16 * 128, C::UM_HALF, 1024),
                                idO, (!first || kk > 0) ? 1u : 0u);
                umma_commit(ub + 8 * (UB_O_DONE + (pv & 1)));
                if (!(pfl[i] & F_LAST)) umma_commit(empty0 + pst[i] * 8);
                ++pv;
                prog = true;
            }
            if (!end) {
                if (!have_md && mbar_test(full0 + stage * 8, phase)) {
                    flags = smeta[stage].flags;
                    have_md = true;
                    if (flags & F_END) end = true;
                }
                if (have_md && !end && k - pv < kPend) {
                    bool ready = true;
                    if (flags & F_FIRST)
                        ready = pv == k && mbar_test(ub + 8 * UB_Q_READY, (uint32_t)(seg & 1));
                    if constexpr (C::KQ) {
                        if (ready) ready = mbar_test(ub + 8 * UB_KDQ, (uint32_t)(k & 1));
                    }
                    if (ready && k > 0) ready = mbar_test(ub + 8 * UB_S_FREE, (uint32_t)((k - 1) & 1));
                    if (ready) {
                        if (flags & F_FIRST) ++seg;
                        tc_fence_after();
                        const uint32_t kb = sbase + stage * C::STAGE_BYTES;
                        const uint32_t qa = tmem + UM_Q + (uint32_t)(((seg - 1) & 1) * 64);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_f16_ts(tmem + UM_S, qa + kk * 8,
                                        smem_desc(kb + (kk >> 2) * C::UM_HALF + (kk & 3) * 32, 16, 1024), idS,
                                        kk > 0 ? 1u : 0u);
                        umma_commit(ub + 8 * UB_S_FULL);
                        pst[k % kPend] = stage;
                        pfl[k % kPend] = flags;
                        ++k;
                        have_md = false;
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                        prog = true;
                    }
                }
            } else if (pv == k) {
                break;
            }
            // watchdog: no progress for the wait limit
            if (prog) {
                idle = 0;
            } else if ((++idle & 1023u) == 0) {
                const uint64_t now = globaltimer_ns();
                if (idle == 1024u) t_idle = now;
                else if (now - t_idle > kWaitLimitNs) ok = false;
            }
        }
        if (!ok) {
            atomicOr(p.err, KV_DEV_TIMEOUT);
            *abort_flag = 1;
        }
        // every MMA issued must have finished before tensor memory is freed
        umma_commit(ub + 8 * UB_DRAIN);
        if (!mbar_wait_bounded(ub + 8 * UB_DRAIN, 0, kWaitLimitNs)) atomicOr(p.err, KV_DEV_TIMEOUT);
    }
    __syncwarp();
}

template <class C>
__global__ void __maxnreg__(C::MAXREG)
    paged_attention_kernel(const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int abort_flag;
    const uint32_t sbase = smem_u32(smem);
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(sbase + C::BAR_OFF + i * 8, 1);
            // the tcgen05 consumer releases a stage with one arrive (an MMA
            // commit, or the merge at a segment end)
            mbar_init(sbase + C::BAR_OFF + (C::STAGES + i) * 8, C::UMR ? 1 : C::NCW);
        }
        if constexpr (C::UMR > 0) {
            const uint32_t ub = sbase + C::UB_OFF;
            const uint32_t counts[10] = {1, 4, 4, 4, 1, 1, 4, 4, 4, 1};  // see the UB_* indices
            for (int i = 0; i < 10; ++i) mbar_init(ub + 8 * i, counts[i]);
        }
        fence_barrier_init();
    }
    // zero the padded query rows of every stage and the zero row
    if constexpr (!C::FMA) {
        const int used = p.pr ? 0 : p.rows * C::QROW;  // head pairs: padding rows inside
        for (int st = 0; st < C::STAGES; ++st) {
            uint8_t* qa = smem + st * C::STAGE_BYTES + C::Q_OFF;
            for (int i = used + threadIdx.x * 16; i < C::RP * C::QROW; i += C::THREADS * 16)
                *reinterpret_cast<uint4*>(qa + i) = make_uint4(0, 0, 0, 0);
        }
    }
    if (threadIdx.x < 8)
        reinterpret_cast<uint4*>(smem + C::ZERO_OFF)[threadIdx.x] = make_uint4(0, 0, 0, 0);
    const int warp = threadIdx.x >> 5;
    if constexpr (C::UMR > 0) {
        // one CTA per SM: all 512 columns
        if (warp == C::NCW + 1) {
            tmem_alloc(sbase + C::TSLOT_OFF, UM_COLS);
            tmem_relinquish();
        }
        tc_fence_before();
    }
    fence_proxy_async();
    __syncthreads();
    pdl_launch_dependents();
    if constexpr (C::UMR > 0) {
        tc_fence_after();
        const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::TSLOT_OFF);
        if (warp == C::NCW)
            producer<C>(&tmK, &tmV, p, smem, &abort_flag);
        else if (warp == C::NCW + 1)
            mma_um<C>(p, smem, tmem, &abort_flag);
        else
            consumer_um<C>(p, smem, tmem, &abort_flag);
        tc_fence_before();
        __syncthreads();
        if (warp == C::NCW + 1) {
            tc_fence_after();
            tmem_dealloc(tmem, UM_COLS);
        }
    } else {
        if (warp == C::NCW) {
            producer<C>(&tmK, &tmV, p, smem, &abort_flag);
        } else if constexpr (C::FMA) {
            consumer_fma<C>(p, smem, &abort_flag);
        } else if constexpr (C::NR8 > 0) {
            consumer_tc<C>(p, smem, &abort_flag);
        } else {
            static_assert(C::MT > 1, "one row tile of more than one row uses the transposed consumer");
            consumer_mma_mt<C>(p, smem, &abort_flag);
        }
    }
}

// ---------------------------------------------------------------------------
// Split-context merge: CTA c merges the (sequence, kv-head) whose last piece
// it computed, from the partials of CTAs meta.first .. c:
//   lse* = log2 sum_i 2^(lse_i),  out = sum_i 2^(lse_i - lse*) o_i.
// One thread per (row, 8 output dims); one pass with a running maximum, two
// pieces per step with all their loads issued together (the kernel is bound
// by the latency of those loads, not by their bytes).
template <int D, int RP>
__global__ void __launch_bounds__(512) lse_merge_kernel(const Params p)
{
    pdl_wait();
    const int c = blockIdx.x;
    const int4 md = p.meta[c];
    if (md.x < 0) return;
    const int idx = threadIdx.x;
    if (idx >= p.rows * (D / 8)) return;
    const int s = md.x, kvh = md.y, a = md.z, slot_a = md.w;
    const int R = idx / (D / 8);
    const int d0 = (idx % (D / 8)) * 8;
    int j = 0;
    const int qh = row_head(p, kvh, R, j);
    if (qh < 0) return;  // a padding row
    float M = kNegInf, W = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = a; i <= c; i += 2) {
        const bool two = i + 1 <= c;
        const int64_t pr0 = ((int64_t)i * 2 + (i == a ? slot_a : 0)) * RP + R;
        const int64_t pr1 = two ? ((int64_t)(i + 1) * 2) * RP + R : pr0;
        const float l0 = p.part_lse[pr0];
        const float l1 = two ? p.part_lse[pr1] : kNegInf;
        const float4* o0 = reinterpret_cast<const float4*>(p.part_o + pr0 * D + d0);
        const float4* o1 = reinterpret_cast<const float4*>(p.part_o + pr1 * D + d0);
        const float4 x0 = o0[0], y0 = o0[1], x1 = o1[0], y1 = o1[1];
        const float mn = fmaxf(M, fmaxf(l0, l1));
        if (mn == kNegInf) continue;  // no visible token so far
        const float f = ex2(M - mn);  // 0 while M is still -inf
        const float w0 = ex2(l0 - mn), w1 = two ? ex2(l1 - mn) : 0.f;
        const float v0[8] = {x0.x, x0.y, x0.z, x0.w, y0.x, y0.y, y0.z, y0.w};
        const float v1[8] = {x1.x, x1.y, x1.z, x1.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = acc[e] * f + w0 * v0[e] + w1 * v1[e];
        W = W * f + w0 + w1;
        M = mn;
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    uint4 v;
    v.x = pack_half2(acc[0] * inv, acc[1] * inv);
    v.y = pack_half2(acc[2] * inv, acc[3] * inv);
    v.z = pack_half2(acc[4] * inv, acc[5] * inv);
    v.w = pack_half2(acc[6] * inv, acc[7] * inv);
    __half* dst = p.out + (((int64_t)s * p.q_len + j) * p.Hq + qh) * D + d0;
    *reinterpret_cast<uint4*>(dst) = v;
}

}  // namespace pkv

// ===========================================================================
// Host side
namespace {

using namespace pkv;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_mu;

struct TmapEntry {
    const void* ptr;
    uint64_t rows;
    int D, BS, dev, int8;
    CUtensorMap map;
};
constexpr int kTmapCache = 32;
TmapEntry g_tmaps[kTmapCache];
int g_tmap_next = 0;

int get_encoder()
{
    if (g_encode) return KV_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return kv_fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return KV_OK;
}

// Tensor map of a pool viewed as [num_blocks*Hkv*BS rows][D] fp16 whose box
// is one (block, kv-head) tile, 128-byte swizzle (kind 0); an int8 code pool
// (kind 1); fp16 with a box of one 64-column half of a tile (kind 2, the
// tcgen05 consumer's layout).  Cached by (pointer, shape, kind, device).
enum : int { TMAP_TILE = 0, TMAP_INT8 = 1, TMAP_HALF = 2 };
int pool_tmap(const void* pool, uint64_t rows, int D, int BS, CUtensorMap* out, int int8 = TMAP_TILE)
{
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(g_mu);
    for (auto& e : g_tmaps)
        if (e.ptr == pool && e.rows == rows && e.D == D && e.BS == BS && e.dev == dev &&
            e.int8 == int8) {
            *out = e.map;
            return KV_OK;
        }
    int rc = get_encoder();
    if (rc != KV_OK) return rc;
    if (int8 == TMAP_HALF) {
        // [rows][D] fp16, box = 64 columns x BS rows (one half of a tile)
        CUtensorMap m;
        const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
        const cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)BS};
        const cuuint32_t estride[2] = {1, 1};
        CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(pool), gdim,
                              gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return kv_fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled failed (half tiles)");
        TmapEntry& e = g_tmaps[g_tmap_next];
        g_tmap_next = (g_tmap_next + 1) % kTmapCache;
        e = {pool, rows, D, BS, dev, int8, m};
        *out = m;
        return KV_OK;
    }
    if (int8 == TMAP_INT8) {
        // int8 code pool as [rows][128]: a box of BS rows is one (block,
        // kv-head) tile of 128-byte rows, 128-byte swizzle
        CUtensorMap m;
        const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
        const cuuint64_t gstride[1] = {(cuuint64_t)D};
        const cuuint32_t box[2] = {(cuuint32_t)D, (cuuint32_t)BS};
        const cuuint32_t estride[2] = {1, 1};
        CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(pool), gdim,
                              gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return kv_fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled failed (int8 K)");
        TmapEntry& e = g_tmaps[g_tmap_next];
        g_tmap_next = (g_tmap_next + 1) % kTmapCache;
        e = {pool, rows, D, BS, dev, int8, m};
        *out = m;
        return KV_OK;
    }
    // The pool as [rows][D/64][64] fp16: a box of BS rows is one whole
    // contiguous (block, kv-head) tile, written with the 128-byte swizzle.
    CUtensorMap m;
    const cuuint32_t rank = D == 64 ? 2 : 3;
    const cuuint64_t gdim[3] = {64, D == 64 ? (cuuint64_t)rows : (cuuint64_t)(D / 64),
                                (cuuint64_t)rows};
    const cuuint64_t gstride[2] = {D == 64 ? (cuuint64_t)128 : (cuuint64_t)128, (cuuint64_t)D * 2};
    const cuuint32_t box[3] = {64, D == 64 ? (cuuint32_t)BS : (cuuint32_t)(D / 64), (cuuint32_t)BS};
    const cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(pool), gdim,
                          gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return kv_fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    TmapEntry& e = g_tmaps[g_tmap_next];
    g_tmap_next = (g_tmap_next + 1) % kTmapCache;
    e = {pool, rows, D, BS, dev, 0, m};
    *out = m;
    return KV_OK;
}

int device_sms()
{
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 1;
}

int rows_padded(int rows) { return rows == 1 ? 1 : 16 * ((rows + 15) / 16); }

size_t workspace_bytes_for(int grid, int rp, int D)
{
    size_t meta = (size_t)grid * 16;
    size_t lse = (size_t)grid * 2 * rp * 4;
    lse = (lse + 15) / 16 * 16;
    size_t po = (size_t)grid * 2 * rp * D * 4;
    return meta + lse + po;
}

template <class C>
int launch(const CUtensorMap& tk, const CUtensorMap& tv, const Params& prm, int grid, bool pdl,
           cudaStream_t stream)
{
    static std::mutex mu;
    static unsigned long long configured = 0;  // bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 64 && !(configured & (1ull << dev))) {
            int rc = kv_cuda_check(
                cudaFuncSetAttribute(paged_attention_kernel<C>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC),
                "cudaFuncSetAttribute");
            if (rc != KV_OK) return rc;
            configured |= 1ull << dev;
        }
    }
    // With PDL the launch may start while the preceding kernel in the stream
    // runs, once that kernel allows it (the library's append kernels do at
    // entry): the set-up (length scan, block-table reads) overlaps its tail,
    // and the loader waits for it before the first read of the pools.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    {
        cudaLaunchConfig_t acfg = {};
        acfg.gridDim = dim3(grid);
        acfg.blockDim = dim3(C::THREADS);
        acfg.dynamicSmemBytes = C::SMEM_ALLOC;
        acfg.stream = stream;
        acfg.attrs = attr;
        acfg.numAttrs = pdl ? 1 : 0;
        int rc = kv_cuda_check(cudaLaunchKernelEx(&acfg, paged_attention_kernel<C>, tk, tv, prm),
                               "paged_attention_kernel launch");
        if (rc != KV_OK) return rc;
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3((unsigned)((prm.rows * (C::D / 8) + 31) / 32 * 32));  // <= 512
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return kv_cuda_check(cudaLaunchKernelEx(&cfg, lse_merge_kernel<C::D, C::RP>, prm),
                         "lse_merge_kernel launch");
}

template <int D, int BS, bool KQ = false>
int dispatch_rows(int rows, bool um, const CUtensorMap& tk, const CUtensorMap& tv, const Params& prm,
                  int grid, bool pdl, cudaStream_t st)
{
    if constexpr (D == 128) {
        // tcgen05 consumer, rows padded to 8, 16 or 32
        if (um) {
            if (rows <= 8) return launch<Cfg<D, BS, 1, false, KQ, 0, 0, 1, 8>>(tk, tv, prm, grid, pdl, st);
            if (rows <= 16) return launch<Cfg<D, BS, 1, false, KQ, 0, 0, 1, 16>>(tk, tv, prm, grid, pdl, st);
            return launch<Cfg<D, BS, 1, false, KQ, 0, 0, 1, 32>>(tk, tv, prm, grid, pdl, st);
        }
    }
    // Tensor-core paths: 128-token stages (8 token warps for one row tile, 4
    // warps of two 16-token sub-tiles for two or three; 256 tokens over int8
    // keys for one row tile or three); more than 24 rows keep the rows-as-M
    // consumer (its accumulators fit 255 registers).
    if (rows == 1) return launch<Cfg<D, BS, 1, true, KQ>>(tk, tv, prm, grid, pdl, st);
    if (rows <= 8) {
        // int8 keys stream 3/4 of the bytes per token: 256-token stages
        if constexpr (KQ) return launch<Cfg<D, BS, 1, false, KQ, 1, 8, 2>>(tk, tv, prm, grid, pdl, st);
        else return launch<Cfg<D, BS, 1, false, KQ, 1, 8, 1>>(tk, tv, prm, grid, pdl, st);
    }
    if (rows <= 16) return launch<Cfg<D, BS, 1, false, KQ, 2, 4, 2>>(tk, tv, prm, grid, pdl, st);
    if (rows <= 24) {
        // int8 keys: 256-token stages (two of them fit the shared memory)
        if constexpr (KQ) return launch<Cfg<D, BS, 1, false, KQ, 3, 4, 4>>(tk, tv, prm, grid, pdl, st);
        else return launch<Cfg<D, BS, 1, false, KQ, 3, 4, 2>>(tk, tv, prm, grid, pdl, st);
    }
    return launch<Cfg<D, BS, 2, false, KQ>>(tk, tv, prm, grid, pdl, st);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Default consumer for several query rows per KV head (head_dim 128): the
// warp-level MMAs, measured faster than the tcgen05 consumer on every
// benchmark shape (8, 20 and 32 rows; fp16 and int8 keys).
bool default_tcgen05(int, bool) { return false; }

// Head pairs: for 8-token blocks (one block of one head is a 2 KB fp16 copy,
// 1 KB of int8 codes; the pair's copies are twice that, half the copies per
// byte) and for int8 keys over 16-token blocks (2 KB of codes), head_dim 128,
// decode (one query), the warp-level consumer; GQA groups of 8 (a row tile
// per head), and over int8 keys also groups of 1, 2 or 4 (a row tile per
// head, partly padding).  Measured: fp16 over 16-token blocks (4 KB copies)
// gains nothing from pairs.
bool pairs_possible(int D, int G, int q_len, int Hkv)
{
    return D == 128 && q_len == 1 && Hkv % 2 == 0 && (G == 1 || G == 2 || G == 4 || G == 8);
}

bool use_head_pairs(int D, int BS, int G, int q_len, int Hkv, bool int8_k, bool um)
{
    if (um || !pairs_possible(D, G, q_len, Hkv)) return false;
    return int8_k || (G == 8 && BS == 8);
}

// Padded query rows of the split partials a launch of this shape may use
// (head pairs take two 8-row tiles whatever the group size).
int rows_padded_for(int G, int q_len, int Hkv, int D)
{
    const int rp = rows_padded(G * q_len);
    return pairs_possible(D, G, q_len, Hkv) && rp < 16 ? 16 : rp;
}

int attention_impl(const void* q, const void* k_pool, const void* v_pool,
                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                   const int32_t* context_lens, int32_t q_len, float scale, void* out, int32_t B,
                   int32_t Hq, int32_t Hkv, int32_t D, int32_t BS, int32_t num_blocks,
                   void* workspace, size_t ws_bytes, const paged_attention_opts* opts,
                   void* stream, const float* k_scale = nullptr)
{
    if (B < 0 || q_len < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || num_blocks < 1 ||
        max_blocks_per_seq < 1)
        return kv_fail(KV_ERR_INVALID, "paged attention: bad sizes");
    if (D != 64 && D != 128) return kv_fail(KV_ERR_INVALID, "paged attention: head_dim must be 64 or 128");
    if (k_scale && D != 128)
        return kv_fail(KV_ERR_INVALID, "paged attention: int8 K pools need head_dim 128");
    if (k_scale && (reinterpret_cast<uintptr_t>(k_scale) & 15u))
        return kv_fail(KV_ERR_INVALID, "paged attention: k_scales must be 16-byte aligned");
    if (BS != 8 && BS != 16) return kv_fail(KV_ERR_INVALID, "paged attention: block_size must be 8 or 16");
    const int G = Hq / Hkv;
    const int rows = G * q_len;
    if (rows > 16 * kMaxMT)
        return kv_fail(KV_ERR_INVALID, "paged attention: (Hq/Hkv)*q_len must be <= 32");
    if ((uint64_t)num_blocks * Hkv * BS >= (1ull << 31))
        return kv_fail(KV_ERR_INVALID, "paged attention: pool too large for 32-bit row coordinates");
    if (B == 0) return KV_OK;
    if (!q || !k_pool || !v_pool || !block_tables || !context_lens || !out || !workspace)
        return kv_fail(KV_ERR_INVALID, "paged attention: null pointer");
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_pool) || !aligned16(v_pool) ||
        !aligned16(workspace))
        return kv_fail(KV_ERR_INVALID, "paged attention: buffers must be 16-byte aligned");
    const int sms = device_sms();
    int grid = sms;
    if (opts && opts->grid_ctas > 0) grid = opts->grid_ctas;
    // consumer for several query rows per KV head at head_dim 128: tcgen05
    // (tensor memory) or warp-level MMAs
    const int consumer = opts ? opts->consumer : 0;
    if (consumer < 0 || consumer > 2)
        return kv_fail(KV_ERR_INVALID, "paged attention: opts.consumer must be 0, 1 or 2");
    const bool um = D == 128 && rows > 1 && (consumer == 2 || (consumer == 0 && default_tcgen05(rows, k_scale != nullptr)));
    // head pairs: the kernel sees Hkv / 2 units of two heads, rows 8h.. of
    // head h, each staged tile both heads' rows of a block (see Cfg::HP)
    const bool hp = use_head_pairs(D, BS, G, q_len, Hkv, k_scale != nullptr, um);
    const int rp = hp ? 16 : rows_padded(rows);
    if (ws_bytes < workspace_bytes_for(grid, rp, D))
        return kv_fail(KV_ERR_INVALID, "paged attention: workspace too small");
    int* err = kv_error_word_ptr();
    if (!err) return kv_fail(KV_ERR_CUDA, "paged attention: no device error word");
    CUtensorMap tk, tv;
    const uint64_t prow = (uint64_t)num_blocks * Hkv * BS;
    const int trows = hp ? 2 * BS : BS;  // pool rows per staged tile
    int rc = pool_tmap(k_pool, prow, D, trows, &tk, k_scale ? TMAP_INT8 : (um ? TMAP_HALF : TMAP_TILE));
    if (rc != KV_OK) return rc;
    rc = pool_tmap(v_pool, prow, D, trows, &tv, um ? TMAP_HALF : TMAP_TILE);
    if (rc != KV_OK) return rc;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    Params prm;
    prm.q = static_cast<const __half*>(q);
    prm.out = static_cast<__half*>(out);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.meta = reinterpret_cast<int4*>(ws);
    size_t off = (size_t)grid * 16;
    prm.part_lse = reinterpret_cast<float*>(ws + off);
    off += ((size_t)grid * 2 * rp * 4 + 15) / 16 * 16;
    prm.part_o = reinterpret_cast<float*>(ws + off);
    prm.err = err;
    prm.k_scale = k_scale;
    prm.max_blocks = max_blocks_per_seq;
    prm.B = B;
    prm.q_len = q_len;
    prm.Hq = Hq;
    prm.Hkv = hp ? Hkv / 2 : Hkv;
    prm.G = G;
    prm.rows = hp ? 16 : rows;
    prm.pr = hp ? rows : 0;
    prm.num_blocks = num_blocks;
    prm.min_share = (opts && opts->min_split_blocks > 0) ? opts->min_split_blocks : 16;
    prm.seg_cost = (opts && opts->seg_cost_blocks != 0) ? (opts->seg_cost_blocks > 0 ? opts->seg_cost_blocks : 0)
                                                        : (k_scale && rows > 1 ? kSegCostTokensQ8 : kSegCostTokens) / BS;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.slot_wait_ns = (opts && opts->producer_wait_ns > 0) ? (uint64_t)opts->producer_wait_ns
                                                            : kWaitLimitNs;
    const bool pdl = !(opts && opts->use_pdl < 0);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (hp) {
        if (!k_scale) return launch<Cfg<128, 8, 1, false, false, 2, 4, 1, 0, 2>>(tk, tv, prm, grid, pdl, st);
        return BS == 8 ? launch<Cfg<128, 8, 1, false, true, 2, 4, 2, 0, 2>>(tk, tv, prm, grid, pdl, st)
                       : launch<Cfg<128, 16, 1, false, true, 2, 4, 2, 0, 2>>(tk, tv, prm, grid, pdl, st);
    }
    if (k_scale)
        return BS == 8 ? dispatch_rows<128, 8, true>(rows, um, tk, tv, prm, grid, pdl, st)
                       : dispatch_rows<128, 16, true>(rows, um, tk, tv, prm, grid, pdl, st);
    if (D == 64) {
        return BS == 8 ? dispatch_rows<64, 8>(rows, false, tk, tv, prm, grid, pdl, st)
                       : dispatch_rows<64, 16>(rows, false, tk, tv, prm, grid, pdl, st);
    }
    return BS == 8 ? dispatch_rows<128, 8>(rows, um, tk, tv, prm, grid, pdl, st)
                   : dispatch_rows<128, 16>(rows, um, tk, tv, prm, grid, pdl, st);
}

}  // namespace

extern "C" {

int paged_attention_workspace_size(int32_t Hq, int32_t Hkv, int32_t q_len, int32_t head_dim,
                                   int32_t grid_ctas, size_t* bytes_out)
{
    if (!bytes_out || Hq < 1 || Hkv < 1 || Hq % Hkv || q_len < 1 ||
        (head_dim != 64 && head_dim != 128))
        return kv_fail(KV_ERR_INVALID, "paged_attention_workspace_size: bad arguments");
    const int rows = (Hq / Hkv) * q_len;
    if (rows > 16 * kMaxMT)
        return kv_fail(KV_ERR_INVALID, "paged_attention_workspace_size: rows must be <= 32");
    const int grid = grid_ctas > 0 ? grid_ctas : device_sms();
    *bytes_out = workspace_bytes_for(grid, rows_padded_for(Hq / Hkv, q_len, Hkv, head_dim), head_dim);
    return KV_OK;
}

int paged_decode_attention(const void* q, const void* k_pool, const void* v_pool,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, float scale, void* out, int32_t B,
                           int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                           int32_t num_blocks, void* workspace, size_t workspace_bytes,
                           void* stream)
{
    return attention_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, 1,
                          scale, out, B, Hq, Hkv, head_dim, block_size, num_blocks, workspace,
                          workspace_bytes, nullptr, stream);
}

int paged_verify_attention(const void* q, const void* k_pool, const void* v_pool,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t q_len, float scale, void* out,
                           int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim,
                           int32_t block_size, int32_t num_blocks, void* workspace,
                           size_t workspace_bytes, void* stream)
{
    return attention_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, q_len,
                          scale, out, B, Hq, Hkv, head_dim, block_size, num_blocks, workspace,
                          workspace_bytes, nullptr, stream);
}

int paged_attention_q8k(const void* q, const void* kq_pool, const float* k_scales,
                        const void* v_pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* context_lens, int32_t q_len, float scale, void* out,
                        int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                        int32_t num_blocks, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!k_scales) return kv_fail(KV_ERR_INVALID, "paged_attention_q8k: null k_scales");
    return attention_impl(q, kq_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, q_len,
                          scale, out, B, Hq, Hkv, head_dim, block_size, num_blocks, workspace,
                          workspace_bytes, nullptr, stream, k_scales);
}

int paged_attention_q8k_ex(const void* q, const void* kq_pool, const float* k_scales,
                           const void* v_pool, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t q_len,
                           float scale, void* out, int32_t B, int32_t Hq, int32_t Hkv,
                           int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           void* workspace, size_t workspace_bytes,
                           const paged_attention_opts* opts, void* stream)
{
    if (!k_scales) return kv_fail(KV_ERR_INVALID, "paged_attention_q8k_ex: null k_scales");
    return attention_impl(q, kq_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, q_len,
                          scale, out, B, Hq, Hkv, head_dim, block_size, num_blocks, workspace,
                          workspace_bytes, opts, stream, k_scales);
}

int paged_attention_ex(const void* q, const void* k_pool, const void* v_pool,
                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, int32_t q_len, float scale, void* out,
                       int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                       int32_t num_blocks, void* workspace, size_t workspace_bytes,
                       const paged_attention_opts* opts, void* stream)
{
    return attention_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, q_len,
                          scale, out, B, Hq, Hkv, head_dim, block_size, num_blocks, workspace,
                          workspace_bytes, opts, stream);
}

}  // extern "C"

// ===========================================================================
// Decode attention with library-owned scratch.
//
// The ordinary entry points take a caller-allocated workspace.  Some callers
// cannot provide one: code that runs where every device byte is handed out by
// someone else's allocator and a stray cudaMalloc is not allowed, plugins that
// get tensors from a host framework but no allocation hook, and latency-
// critical paths where a cudaMalloc (which may synchronise the device) must
// never happen after start-up.  For them the split-context scratch lives in
// this fixed array, loaded with the library: every GPU that loads the library
// holds kStaticScratchBytes of it until the process exits.
namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;  // 8 MiB
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
void* g_static_scratch_ptr[kMaxScratchDevices];
std::mutex g_static_scratch_mu;

// Device address of this device's copy of the array.  In host code the
// array's name is only a host-side stand-in; the real address comes from the
// runtime, looked up once per device with that device current.
int static_scratch_address(void** out)
{
    int dev = 0;
    int rc = kv_cuda_check(cudaGetDevice(&dev), "paged_decode_attention_static_ws");
    if (rc != KV_OK) return rc;
    if (dev < 0 || dev >= kMaxScratchDevices)
        return kv_fail(KV_ERR_INVALID, "paged_decode_attention_static_ws: device index too large");
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    if (!g_static_scratch_ptr[dev]) {
        void* p = nullptr;
        rc = kv_cuda_check(cudaGetSymbolAddress(&p, g_static_scratch),
                           "paged_decode_attention_static_ws: cudaGetSymbolAddress");
        if (rc != KV_OK) return rc;
        g_static_scratch_ptr[dev] = p;
    }
    *out = g_static_scratch_ptr[dev];
    return KV_OK;
}

}  // namespace

extern "C" int paged_decode_attention_static_ws(const void* q, const void* k_pool,
                                                const void* v_pool, const int32_t* block_tables,
                                                int32_t max_blocks_per_seq,
                                                const int32_t* context_lens, float scale,
                                                void* out, int32_t B, int32_t Hq, int32_t Hkv,
                                                int32_t head_dim, int32_t block_size,
                                                int32_t num_blocks, void* stream)
{
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (head_dim != 64 && head_dim != 128))
        return kv_fail(KV_ERR_INVALID, "paged_decode_attention_static_ws: bad sizes");
    const int rows = Hq / Hkv;
    if (rows > 16 * kMaxMT)
        return kv_fail(KV_ERR_INVALID, "paged_decode_attention_static_ws: Hq/Hkv must be <= 32");
    const size_t need = workspace_bytes_for(device_sms(), rows_padded_for(rows, 1, Hkv, head_dim), head_dim);
    if (need > kStaticScratchBytes)
        return kv_fail(KV_ERR_INVALID,
                       "paged_decode_attention_static_ws: this shape needs more scratch than the "
                       "library's fixed 8 MiB; use paged_decode_attention with a workspace");
    void* scratch = nullptr;
    const int rc = static_scratch_address(&scratch);
    if (rc != KV_OK) return rc;
    return attention_impl(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, 1,
                          scale, out, B, Hq, Hkv, head_dim, block_size, num_blocks, scratch,
                          kStaticScratchBytes, nullptr, stream);
}
