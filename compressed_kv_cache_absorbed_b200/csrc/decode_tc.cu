// Absorbed MLA decode on the tcgen05 tensor cores, for H = 128 heads, d_c = 512, d_hR = 64.
//
// Problem (per sequence b, head h, cached token t; scale = 1/sqrt(192)):
//     s[h,t] = scale * ([q_lat | q_rope][h] . [c_t | k_r,t])      (576-long dot product)
//     o_lat[h] = sum_t softmax_t(s[h,:]) c_t                       (512 wide)
// With 128 heads sharing every cache row this is a dense contraction: per 64-token tile,
// S = Q[128 x 576] . tile^T and O += P[128 x 64] . tile[:, :512].
//
// Why two CTAs per tile.  O for 128 heads x 512 latent columns in fp32 is 512 TMEM columns,
// all of an SM's TMEM.  So a cluster of two CTAs (two SMs) splits the latent columns: CTA r
// owns c columns [256r, 256r + 256) and rotary columns [32r, 32r + 32), loads only those
// (no duplicate HBM/L2 traffic, no multicast), and accumulates O_r = 128 x 256.  The
// softmax needs the full 576-long scores, so each CTA computes a partial S_r over its 288
// columns and the pair swaps them through distributed shared memory (one 16 KB bulk copy
// per tile, bf16 partials); both CTAs then run the same softmax for all 128 heads,
// which costs 64 exponentials per thread per tile and saves a second exchange hop.
//
// TMEM of one CTA (512 columns x 128 lanes; lane = head):
//     [0, 128)   Q_r latent part as the MMA A operand (256 bf16, two per column)
//     [128, 192) S_r partial scores, fp32, 64 tokens
//     [192, 256) P probabilities as the A operand, two buffers of 64 bf16 (tile g uses g & 1)
//     [256, 512) O_r accumulator, fp32
// The 32 rotary query columns of the CTA live in shared memory (64-byte swizzle) and enter
// the score MMA as an SS operand; that frees the TMEM for the second P buffer, so the
// softmax of tile g + 1 does not wait for the O MMAs of tile g.  The latent score MMAs and
// the O MMAs read A from TMEM and only the tile from shared memory.
//
// Warp roles (480 threads): warp 0 issues TMA loads of 64-token tiles (4 latent boxes of
// 64 columns with 128-byte swizzle + this CTA's 32 rotary columns with 64-byte swizzle,
// 36 KB) into a 5-stage ring; warp 1 owns TMEM and issues the score MMAs, warp 14 the
// P c MMAs (FP8 rows: warp 1 issues both, warps 14-15 dequantise); warps 2-5 (thread = head
// = TMEM lane) load Q and send partial scores to the peer; warps 6-13 (two per TMEM
// subpartition, one per half tile) run the online softmax (base-2, lazy rescale: the running
// max moves only when a tile exceeds it by more than 8, so p <= 256), write P, and read O
// back at the end of each piece.
//
// Work split: the tiles of all sequences, in order, are cut into equal ranges, one per
// cluster; a range may hold pieces of several sequences.  Each piece writes an
// partial (its normalised output O / l in fp16, its running max and row sum) that the merge
// kernel combines.
// Every wait is bounded; a timeout latches an error and the kernel drains and exits.
#include <math.h>

#include "common.cuh"
#include "decode_tc.cuh"
#include "tc_common.cuh"

namespace mla {
namespace tc {

namespace {

constexpr int kT = 64;                        // tokens per tile
constexpr int kChunkBytes = kT * 128;         // one 64-column latent box of a tile (128-byte swizzle)
constexpr int kRopeBytes = kT * 64;           // this CTA's 32 rotary columns of a tile (64-byte swizzle)
constexpr int kTileBytes = 4 * kChunkBytes + kRopeBytes;
constexpr int kQRopeBytes = 128 * 64;         // this CTA's 32 rotary query columns, 128 heads
constexpr int kXRowBytes = kT * 2;            // one head's 64 bf16 partial scores (128 B)
constexpr int kXBytes = 128 * kXRowBytes;     // one exchange buffer: 128 heads x 64 tokens
constexpr int kBarBytes = 256 + 2048 + 256;
// FP8 cache rows (see decode_tc.cuh): per tile and CTA, this CTA's 256 codes (two 128-byte
// boxes, 128-byte swizzle), its 32 rotary columns (bf16, 64-byte swizzle) and the 64 rows'
// 16-byte scale fields (the fp32 scale first).  They land in place in a stage the size of a
// bf16 tile: the codes in the upper half of the latent area (fp16 boxes 2 and 3), the rotary
// box where the tile keeps it, the scales at the start of fp16 box 0 (read before box 0 is
// written); the dequantisation warps then expand the codes into the four fp16 latent boxes.
constexpr int kF8CodeBytes = kT * 128;
constexpr int kF8CodeOffset = 2 * kChunkBytes;        // code boxes at fp16 boxes 2, 3
constexpr int kF8StageScaleOffset = 0;                 // in fp16 box 0, written last
constexpr int kF8TileBytes = kTileBytes;               // 36 KB
constexpr int kF8LoadBytes = 2 * kF8CodeBytes + kRopeBytes + kT * 16;
static_assert(kF8TileBytes % 1024 == 0, "FP8 stages keep the 1024-byte alignment of the swizzled boxes");

// Two variants of the kernel.  bf16 cache rows: TMA fills a ring of kStages tiles that the
// MMAs read directly.  FP8 cache rows: TMA fills each stage with FP8 data and two
// dequantisation warps turn it in place into an fp16 tile (code x scale) of the same layout;
// the latent MMAs then run on fp16 operands (q_lat and P in fp16 too).
template <bool kF8> struct DecCfg;
// kSplitIssue: the score MMAs and the P c MMAs are issued by two threads in different warps
// (warp 1 and warp 14), each waiting only for its own operands, so a ready P is not held up
// behind the issue of the next score batch.  Otherwise one thread issues both (warp 1).
// Both variants: 5 stages and one partial-score exchange buffer per direction (a fifth stage
// fits only beside one buffer).  With 4 stages the next score batch often waited for its
// tile to land; the ring, not the exchange, held the score MMAs back.
template <> struct DecCfg<false> {
    static constexpr int kStages = 5, kStageBytes = kTileBytes, kXBufs = 1;
    static constexpr int kThreads = 480;   // producer, S issuer, 4 sender, 8 softmax warps, P c issuer
    static constexpr bool kSplitIssue = true;
};
template <> struct DecCfg<true> {
    static constexpr int kStages = 5, kStageBytes = kF8TileBytes, kXBufs = 1;
    static constexpr int kThreads = 512;   // producer, MMA, 4 sender, 8 softmax, 2 dequantisation warps
    static constexpr bool kSplitIssue = false;
};
// Shared memory: the ring of kStages tiles, kXBufs receive buffers for the peer's partial
// scores and kXBufs staging buffers for this CTA's own (each kXBytes).  The
// dynamic shared memory of a kernel without static shared memory starts 1024-byte aligned
// (the 128-byte swizzle needs it); the kernel checks this instead of padding.
template <bool kF8>
constexpr int dec_smem() {
    return DecCfg<kF8>::kStages * DecCfg<kF8>::kStageBytes + 2 * DecCfg<kF8>::kXBufs * kXBytes + kQRopeBytes +
           kBarBytes;
}
static_assert(dec_smem<false>() <= 232448, "decode kernel shared memory over the 227 KB limit");
// The barrier area: tile_full and tile_empty [kStages], 20 single barriers from s_full on,
// f8_full [kStages], the pair's 2 x 2 x 128 floats, then the TMEM slot, the abort flag and
// the planning's 16 + 2 ints.
template <bool kF8>
constexpr int dec_bar_bytes() { return (3 * DecCfg<kF8>::kStages + 20) * 8 + 512 * 4 + (2 + 16 + 2) * 4; }
static_assert(dec_bar_bytes<false>() <= kBarBytes && dec_bar_bytes<true>() <= kBarBytes,
              "decode kernel barrier area over its reserved bytes");
static_assert(dec_smem<true>() <= 232448, "FP8 decode kernel shared memory over the 227 KB limit");
constexpr uint32_t kColQ = 0, kColS = 128, kColP = 192, kColO = 256, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

// The work split counts cost units: one per tile plus kPieceCost for every sequence start
// (a new piece costs its partial's epilogue and a query reload: a switch stalls the score
// MMAs ~4.5 us, about five 64-token tiles), so clusters whose range starts sequences get
// fewer tiles.  Tile j of sequence b sits at cost position first[b] + j, with first[b] =
// (cost of all earlier sequences) + kPieceCost.
constexpr int kPieceCost = 5;

// The merge kernel recomputes this split from the offsets (it needs each sequence's first
// and last cost positions and the cost units per cluster).

__device__ __forceinline__ int tiles_of_len(int L) { return L > 0 ? (L + kT - 1) / kT : 0; }
__device__ __forceinline__ int cost_of_tiles(int n) { return n > 0 ? n + kPieceCost : 0; }

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// 2^x with the hardware approximation (inputs here are <= 8; results below 2^-126 flush to 0)
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A piece of work: tiles [j0, j1) of parent sequence b (whose rows start at row0 or sit in
// b's pages) for query v, which attends to the first L of b's rows.
struct Seg {
    int b, v, j0, j1, L, slot;
    long long row0;
};

// Where the cache rows of a sequence live: rows [offsets[b], offsets[b+1]) of the cache, or,
// with a block table (paged cache), seq_lens[b] tokens in 64-token pages, tile j of sequence
// b in page block_table[b * bt_stride + j] (cache rows 64 page .. 64 page + 63).
//
// A sequence whose rows are not inside the cache (decreasing or negative offsets, rows past
// cache_rows, more tokens than its block-table row has pages for) is invalid: raw_len
// returns -1 for it, the planner latches MLA_ERR_OUT_OF_RANGE, and every role of both
// kernels sees it as empty (len = 0), so its output is zero and no CTA has to abort.
struct SeqSrc {
    const int32_t* offsets;
    const int32_t* seq_lens;
    const int32_t* block_table;
    int bt_stride;
    long long cache_rows;
    __device__ int raw_len(int b) const {
        if (block_table) {
            const int L = seq_lens[b];
            return (L < 0 || (long long)L > (long long)bt_stride * 64) ? -1 : L;
        }
        const long long r0 = offsets[b], r1 = offsets[b + 1];
        return (r0 < 0 || r1 < r0 || r1 > cache_rows) ? -1 : (int)(r1 - r0);
    }
    __device__ int len(int b) const {
        const int L = raw_len(b);
        return L > 0 ? L : 0;
    }
    __device__ long long row0(int b) const { return block_table ? 0 : offsets[b]; }
};

// Walks the pieces of sequences in this cluster's cost range [lo, hi), in sequence order,
// starting from the sequence whose cost region holds lo (cost start cs).  The same walk runs
// in every role of both CTAs.
//
// Sibling queries.  With Q > 1, each sequence b carries Q queries (the last Q rows of b are
// new tokens; query v = b Q + t attends to the first len(b) - (Q - 1 - t) rows).  The
// clusters form groups of Q siblings: cluster c takes cost range c / Q of the sequences and
// query t = c % Q, so the Q siblings walk the same tiles at the same time and the cache
// streams from HBM once while L2 serves the other Q - 1 reads.  Costs are counted on the
// sequences, so all siblings get the same ranges; a sibling whose query ends earlier skips
// the tiles past its end.
//
// Partial slots: a piece that starts at its query's first tile takes slot v; the one piece
// of a cluster that continues a query begun in an earlier range takes slot B Q + cluster.
// So B Q + clusters slots suffice.
template <bool kSib>
struct SegIter {
    SeqSrc src;
    int B, lo, hi, cluster, b, cs;
    int Qr, tr;   // siblings and this cluster's query (used with kSib only)
    __device__ __forceinline__ int Q() const { return kSib ? Qr : 1; }
    __device__ __forceinline__ int t() const { return kSib ? tr : 0; }
    __device__ bool next(Seg& s) {
        const int Q = this->Q(), t = this->t();
        while (b < B && cs < hi) {
            const int L = src.len(b);
            const long long r0 = src.row0(b);
            const int n = tiles_of_len(L);
            const int f = cs + kPieceCost;   // cost position of tile 0
            const int bb = b;
            ++b;
            cs += cost_of_tiles(n);
            if (n == 0) continue;
            const int Lt = L - (Q - 1 - t);    // rows this query attends to
            const int nt = tiles_of_len(Lt);
            const int j0 = lo > f ? lo - f : 0;
            const int j1 = hi - f < nt ? hi - f : nt;
            if (j0 < j1) {
                s.b = bb;
                s.v = bb * Q + t;
                s.j0 = j0;
                s.j1 = j1;
                s.row0 = r0;
                s.L = Lt;
                s.slot = j0 == 0 ? s.v : B * Q + cluster;
                return true;
            }
        }
        return false;
    }
};

__device__ __forceinline__ void fail(int* code, long long* detail, volatile int* abort_flag, int where) {
    latch(DevErr{code, detail}, kErrTimeout, (long long)where * 1000000 + blockIdx.x);
    *abort_flag = 1;
}

// FP8 -> fp16 of 16 codes (one 16-byte unit), each times the row's scale (fp16)
__device__ __forceinline__ void dequant16(const uint4 c, __half2 s, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t a, b;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(a) : "h"((unsigned short)(w[i] & 0xFFFFu)));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(b) : "h"((unsigned short)(w[i] >> 16)));
        __half2 ha = __hmul2(*reinterpret_cast<__half2*>(&a), s);
        __half2 hb = __hmul2(*reinterpret_cast<__half2*>(&b), s);
        o[2 * i] = *reinterpret_cast<uint32_t*>(&ha);
        o[2 * i + 1] = *reinterpret_cast<uint32_t*>(&hb);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

template <bool kF8, bool kSib>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(DecCfg<kF8>::kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_cache, const __grid_constant__ CUtensorMap tm_rope,
                 const __grid_constant__ CUtensorMap tm_scale,
                 const __nv_bfloat16* __restrict__ q_lat,
                 const __nv_bfloat16* __restrict__ q_rope, long long sQr_b, long long sQr_h,
                 const SeqSrc src, int B, int Q_arg, int stream_once, long long cache_rows,
                 float scale_log2,
                 __half* __restrict__ part_o, float* __restrict__ part_ml, const uint8_t* __restrict__ next_weights,
                 long long next_weight_bytes, int* err_code, long long* err_detail) {
    constexpr int kStages = DecCfg<kF8>::kStages, kStride = DecCfg<kF8>::kStageBytes;
    const int Q = kSib ? Q_arg : 1;   // queries per sequence (sibling clusters)
    constexpr int kThreads = DecCfg<kF8>::kThreads;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (ptx::smem_u32(smem_raw) & 1023) {   // uniform across the CTA: leave before any sync
        if (threadIdx.x == 0) latch(DevErr{err_code, err_detail}, kErrTimeout, 7000000);
        return;
    }
    // this thread's sequence length for the planning below, requested before the set-up
    // so that the load overlaps it
    const int len0 = threadIdx.x < B ? src.raw_len(threadIdx.x) : 0;
    uint8_t* smem = smem_raw;
    uint8_t* tiles = smem;
    constexpr uint32_t kXB = DecCfg<kF8>::kXBufs;
    uint8_t* xbuf = smem + kStages * kStride;      // [kXB] partial scores received from the peer
    uint8_t* xstage = xbuf + kXB * kXBytes;        // [kXB] this CTA's partial scores, being sent
    uint8_t* qrope = xstage + kXB * kXBytes;       // rotary query columns (A operand, 64-byte swizzle)
    uint64_t* bars = (uint64_t*)(qrope + kQRopeBytes);
    uint64_t* tile_full = bars;
    uint64_t* tile_empty = bars + kStages;
    uint64_t* s_full = bars + 2 * kStages;
    uint64_t* s_free = s_full + 1;
    uint64_t* p_ready = s_full + 2;    // [2] P of tile g is in P buffer g & 1
    uint64_t* o_done = s_full + 4;     // [2] the O MMAs of tile g (and all before) completed
    uint64_t* q_ready = s_full + 6;
    // [kXB] the peer's partial scores for tile g landed in xbuf[g % kXB]: armed locally with
    // the byte count, completed by the peer's bulk copy
    uint64_t* x_full = s_full + 7;
    // [kXB] the peer has read what this CTA sent into its xbuf[g % kXB]; that copy therefore
    // also finished reading this CTA's xstage[g % kXB] (one arrive per peer warp)
    uint64_t* x_empty = s_full + 9;
    uint64_t* drain = s_full + 11;     // all MMAs issued by this CTA have completed
    uint64_t* xs_ready = s_full + 12;  // [kXB] all 128 rows of xstage[g % kXB] written
    uint64_t* xs_free = s_full + 14;   // [kXB] the local softmax has read xstage[g % kXB]
    uint64_t* pair_bar = s_full + 16;  // [4] the two softmax warps of a subpartition
    uint64_t* f8_full = s_full + 20;   // [kStages] a stage's FP8 data landed (FP8 rows)
    float* pair_val = (float*)(f8_full + kStages);   // [2][2][128] values the two warps swap
    uint32_t* tmem_slot = (uint32_t*)(pair_val + 512);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
    int* plan_wsum = (int*)(tmem_slot + 2);   // [16] per-warp sums of the planning scans
    int* plan_first = plan_wsum + 16;         // [2] sequence holding this cluster's first tile, its first tile

    const uint32_t rank = cluster_rank(), peer = rank ^ 1;
    const int cluster = (int)cluster_id_x();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&tile_full[s], kF8 ? 64 : 1);   // the dequantisation warps, or TMA
            ptx::mbar_init(&tile_empty[s], 1);
        }
        if (kF8)
            for (int s = 0; s < kStages; ++s) ptx::mbar_init(&f8_full[s], 1);
        ptx::mbar_init(s_full, 1);
        ptx::mbar_init(s_free, 128);
        ptx::mbar_init(&p_ready[0], 256);
        ptx::mbar_init(&p_ready[1], 256);
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&pair_bar[i], 64);
        ptx::mbar_init(&o_done[0], 1);
        ptx::mbar_init(&o_done[1], 1);
        ptx::mbar_init(q_ready, 128);
        ptx::mbar_init(drain, DecCfg<kF8>::kSplitIssue ? 2 : 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&x_full[i], 1);
            ptx::mbar_init(&x_empty[i], 8);
            ptx::mbar_init(&xs_ready[i], 128);
            ptx::mbar_init(&xs_free[i], 256);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the peer's barriers exist before anyone arrives on them remotely
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) pdl_trigger();

    // ---------------------------------------------------------------- planning
    // Each CTA cuts the tiles of all sequences (in order) into equal ranges itself, from
    // the offsets alone, so the cache loads start without waiting for another kernel.  The
    // call's first kernel waits for all earlier work before it lets this kernel launch, so
    // the offsets and the cache are final; only the absorbed queries (q_lat) come from a
    // kernel of this call, and only the threads that read them wait for it (pdl_wait).
    constexpr int kWarps = kThreads / 32;
    const int P = (int)(gridDim.x / 2);
    int total = 0;
    {
        int mine = 0;
        for (int b = threadIdx.x; b < B; b += kThreads) {
            const int L = b == (int)threadIdx.x ? len0 : src.raw_len(b);
            if (L < 0 && blockIdx.x == 0) latch(DevErr{err_code, err_detail}, kErrOutOfRange, b);
            mine += cost_of_tiles(tiles_of_len(L));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
        if (lane == 0) plan_wsum[warp] = mine;
        if (threadIdx.x == 0) {
            plan_first[0] = B;
            plan_first[1] = 0;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kWarps; ++i) total += plan_wsum[i];
        __syncthreads();
    }
    // Q sibling clusters per cost range (one per query of a sequence); clusters past the
    // last full group of Q have no range
    const int R = P / Q, range = cluster / Q, tok = cluster % Q;
    const int per = total > 0 ? (total + R - 1) / R : 1;
    const int lo = range < R ? range * per : total, hi = min(total, lo + per);
    if (lo < total) {
        int carry = 0;
        for (int c0 = 0; c0 < B; c0 += kThreads) {
            const int b = c0 + (int)threadIdx.x;
            const int n = b < B ? tiles_of_len(c0 == 0 ? len0 : src.len(b)) : 0;
            const int cb = cost_of_tiles(n);
            int incl = cb;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (lane == 31) plan_wsum[warp] = incl;
            __syncthreads();
            int before = carry, chunk = 0;
#pragma unroll
            for (int i = 0; i < kWarps; ++i) {
                const int v = plan_wsum[i];
                before += i < warp ? v : 0;
                chunk += v;
            }
            const int cs = before + incl - cb;   // cost of the sequences before b
            if (b < B) {
                if (cb > 0 && cs <= lo && lo < cs + cb) {   // unique: the cost region holding lo
                    plan_first[0] = b;
                    plan_first[1] = cs;
                }
            }
            carry += chunk;
            __syncthreads();
        }
    }
    SegIter<kSib> it{src, B, lo, hi, cluster, plan_first[0], plan_first[1], Q, tok};
    Seg sg;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // bf16 rows complete the tile itself; FP8 rows complete f8_full, on which the
            // dequantisation warps wait
            constexpr int NR = kStages;
            constexpr int kRingBytes = kF8 ? kF8LoadBytes : kTileBytes;
            uint8_t* ring = tiles;
            uint64_t* ring_full = kF8 ? f8_full : tile_full;
            uint64_t* ring_empty = tile_empty;
            ptx::tma_prefetch(&tm_cache);
            ptx::tma_prefetch(&tm_rope);
            if (kF8) ptx::tma_prefetch(&tm_scale);
            // a cache read once is let go from L2 first, keeping the partials and weights; with
            // sibling queries (or other calls' queries) reading the same tiles it is kept
            const uint64_t stream_policy = stream_once ? ptx::policy_evict_first() : ptx::policy_evict_normal();
            uint32_t g = 0;
            while (!*abort_flag && it.next(sg)) {
                for (int j = sg.j0; j < sg.j1; ++j, ++g) {
                    const int s = g % NR;
                    const uint32_t n = g / NR;
                    if (g >= (uint32_t)NR && !ptx::mbar_wait(&ring_empty[s], (n - 1) & 1, abort_flag)) {
                        fail(err_code, err_detail, abort_flag, 1);
                        break;
                    }
                    uint8_t* dst = ring + s * kStride;
                    long long row_l = sg.row0 + (long long)j * kT;
                    if (src.block_table) {
                        const long long page = src.block_table[(long long)sg.b * src.bt_stride + j];
                        if (page < 0 || (page + 1) * kT > cache_rows) {
                            // a page outside the cache: latch the error and load a tile that
                            // lies wholly past the tensor's last row, which TMA fills with
                            // zeros, so every role still sees the tile it expects
                            latch(DevErr{err_code, err_detail}, kErrOutOfRange, sg.b);
                            row_l = cache_rows;
                        } else {
                            row_l = page * kT;
                        }
                    }
                    const int row = (int)row_l;
                    ptx::mbar_expect_tx(&ring_full[s], kRingBytes);
                    if (kF8) {
                        // this CTA's 256 codes (bytes 256 rank ..), its 32 rotary columns (bf16
                        // elements 256 + 32 rank ..) and the scale fields (fp32 element 160)
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            ptx::tma_load_2d_hint(dst + kF8CodeOffset + i * kF8CodeBytes, &tm_cache, &ring_full[s],
                                                  256 * (int)rank + 128 * i, row, stream_policy);
                        ptx::tma_load_2d_hint(dst + 4 * kChunkBytes, &tm_rope, &ring_full[s], 256 + 32 * (int)rank,
                                              row, stream_policy);
                        ptx::tma_load_2d_hint(dst + kF8StageScaleOffset, &tm_scale, &ring_full[s], 160, row, stream_policy);
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            ptx::tma_load_2d_hint(dst + i * kChunkBytes, &tm_cache, &ring_full[s],
                                                  256 * (int)rank + 64 * i, row, stream_policy);
                        ptx::tma_load_2d_hint(dst + 4 * kChunkBytes, &tm_rope, &ring_full[s], 512 + 32 * (int)rank,
                                              row, stream_policy);
                    }
                }
            }
            // All tiles requested: pull this CTA's share of the next kernel's weights (W_UV)
            // into L2 while the last tiles are processed.
            if (next_weights != nullptr && next_weight_bytes > 0) {
                const long long share = ((next_weight_bytes + gridDim.x - 1) / gridDim.x + 15) & ~15LL;
                const long long a = share * blockIdx.x;
                const long long e = min(next_weight_bytes, a + share);
                const uint64_t keep = ptx::policy_evict_last();
                for (long long o = a; o < e; o += 16384)
                    ptx::bulk_prefetch_l2(next_weights + o, (uint32_t)min(16384LL, e - o), keep);
            }
            // loads still in flight after an abort complete before the CTA leaves
            for (uint32_t k = 0; k < (uint32_t)NR && k < g; ++k) {
                const uint32_t gg = g - 1 - k;
                ptx::mbar_wait(&ring_full[gg % NR], (gg / NR) & 1, nullptr);
            }
        }
    } else if (kF8 && warp >= 14) {
        // ------------------------------------------------- FP8 dequantisation (FP8 rows)
        // 64 threads expand the FP8 data of stage g % kStages in place into its fp16 tile:
        // every 16 codes of a row (one 16-byte unit of a 128-byte-swizzled code box) times the
        // row's scale become two 16-byte units of a 128-byte-swizzled fp16 latent box.  Code
        // box 0 (in fp16 box 2's place) becomes fp16 boxes 0 and 1, which it does not overlap;
        // code box 1 (in fp16 box 3's place) is read into registers by all 64 threads before
        // any of them writes fp16 boxes 2 and 3 over both code boxes.  The rotary box landed
        // where the tile keeps it.
        const int dt = threadIdx.x - 14 * 32;
        uint32_t g = 0;
        bool ok = true;
        Seg cur;
        // unit e = dt + 64 k of code box `box`, row r = e / 8, whose scale is sc
        auto expand = [&](uint8_t* tl, int k, uint4 c, int box, float sc) {
            const int e = dt + 64 * k;
            const int r = e >> 3, u = e & 7, sw = r & 7;       // row, unit within the code box
            uint4 lo, hi;
            dequant16(c, __float2half2_rn(sc), lo, hi);
            // latent columns 128 box + 16 u .. + 15: fp16 box 2 box + (u >> 2), units 2 (u & 3), + 1
            uint8_t* rowp = tl + (2 * box + (u >> 2)) * kChunkBytes + r * 128;
            const int a = 2 * (u & 3);
            *(uint4*)(rowp + ((a ^ sw) << 4)) = lo;
            *(uint4*)(rowp + (((a + 1) ^ sw) << 4)) = hi;
        };
        auto code_unit = [&](const uint8_t* tl, int k, int box) {
            const int e = dt + 64 * k;
            const int r = e >> 3, u = e & 7;
            return *(const uint4*)(tl + kF8CodeOffset + box * kF8CodeBytes + r * 128 + ((u ^ (r & 7)) << 4));
        };
        while (ok && !*abort_flag && it.next(cur)) {
            for (int j = cur.j0; j < cur.j1; ++j, ++g) {
                const int s = g % kStages;
                if (!ptx::mbar_wait(&f8_full[s], (g / kStages) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* tl = tiles + s * kStride;
                float sc[8];   // the scales of this thread's rows (dt / 8 + 8 k), both code boxes
#pragma unroll
                for (int k = 0; k < 8; ++k) sc[k] = *(const float*)(tl + kF8StageScaleOffset + ((dt + 64 * k) >> 3) * 16);
                ptx::named_barrier_sync(8, 64);   // every scale is read before fp16 box 0 covers them
#pragma unroll
                for (int k = 0; k < 8; ++k) expand(tl, k, code_unit(tl, k, 0), 0, sc[k]);
                uint4 c1[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) c1[k] = code_unit(tl, k, 1);
                ptx::named_barrier_sync(8, 64);   // every code of the stage is read
#pragma unroll
                for (int k = 0; k < 8; ++k) expand(tl, k, c1[k], 1, sc[k]);
                ptx::fence_proxy_async_smem();   // read by the tensor cores
                ptx::mbar_arrive(&tile_full[s]);
            }
        }
        if (!ok) fail(err_code, err_detail, abort_flag, 6);
    } else if (DecCfg<kF8>::kSplitIssue && (warp == 1 || warp == 14)) {
        // ------------------------------------------- MMA issuers: S (warp 1), P c (warp 14)
        if (lane == 0) {
            constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(128, kT, 0, 0);
            constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(128, 256, 0, 1);
            uint32_t g = 0, sidx = 0;
            bool ok = true;
            Seg sq;
            SegIter<kSib> iq = it;
            while (ok && !*abort_flag && iq.next(sq)) {
                for (int j = sq.j0; j < sq.j1; ++j, ++g) {
                    const int st = g % kStages;
                    if (warp == 1) {
                        // S of tile g: its tile has landed, S(g - 1) has been read, and at a piece's
                        // first tile the piece's query is in TMEM
                        if (j == sq.j0) {
                            if (!ptx::mbar_wait(q_ready, sidx & 1, abort_flag)) { ok = false; break; }
                            ++sidx;
                        }
                        if (!ptx::mbar_wait(&tile_full[st], (g / kStages) & 1, abort_flag) ||
                            (g > 0 && !ptx::mbar_wait(s_free, (g - 1) & 1, abort_flag))) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t t = ptx::smem_u32(tiles + st * kStride);
#pragma unroll
                        for (int ks = 0; ks < 16; ++ks)   // latent columns: 4 chunks x 4 K-steps
                            ptx::mma_ts(tmem + kColS, tmem + kColQ + 8 * ks,
                                        ptx::desc_kmajor_sw128(t + (ks >> 2) * kChunkBytes + (ks & 3) * 32), idesc_s,
                                        ks != 0);
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks)    // this CTA's half of the rotary columns
                            ptx::mma_ss(tmem + kColS, ptx::desc_kmajor_sw64(ptx::smem_u32(qrope) + 32 * ks),
                                        ptx::desc_kmajor_sw64(t + 4 * kChunkBytes + 32 * ks), idesc_s, 1);
                        ptx::mma_commit(s_full);
                    } else {
                        // O += P c of tile g once its P is in TMEM (the softmax writes a piece's
                        // first P only after reading the previous piece's O)
                        if (!ptx::mbar_wait(&p_ready[g & 1], (g >> 1) & 1, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
                        const uint32_t v = ptx::smem_u32(tiles + st * kStride);
                        const bool first = (j == sq.j0);
#pragma unroll
                        for (int k = 0; k < kT / 16; ++k)
                            ptx::mma_ts(tmem + kColO, tmem + kColP + 32 * (g & 1) + 8 * k,
                                        ptx::desc_mnmajor_sw128(v + 2048 * k, kChunkBytes), idesc_o,
                                        !(first && k == 0));
                        ptx::mma_commit(&o_done[g & 1]);
                        ptx::mma_commit(&tile_empty[st]);
                    }
                }
            }
            if (!ok) fail(err_code, err_detail, abort_flag, 2);
            // drain: wait (bounded) until the MMAs of both issuers have completed
            ptx::mma_commit(drain);
            if (!ptx::mbar_wait(drain, 0, nullptr)) fail(err_code, err_detail, abort_flag, 4);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            // the latent scores and P c: bf16 operands, or fp16 for FP8 rows; the rotary scores bf16
            constexpr uint32_t idesc_s = kF8 ? ptx::idesc_f16_f32(128, kT, 0, 0) : ptx::idesc_bf16_f32(128, kT, 0, 0);
            constexpr uint32_t idesc_sr = ptx::idesc_bf16_f32(128, kT, 0, 0);
            constexpr uint32_t idesc_o = kF8 ? ptx::idesc_f16_f32(128, 256, 0, 1) : ptx::idesc_bf16_f32(128, 256, 0, 1);
            uint32_t g = 0, sidx = 0;
            bool ok = true;
            // Event-driven issue: O of the oldest tile as soon as its P is in TMEM (it frees the
            // P columns for the next tile and the tile's shared-memory stage), otherwise S of
            // the next tile as soon as that tile has landed and the S columns are free.  S may
            // run ahead of O by as many tiles as the ring holds.  Tiles are taken in one flat
            // pass over all pieces (two iterators: one for S, one for O).
            SegIter<kSib> its = it;
            Seg ss;
            bool s_have = !*abort_flag && its.next(ss);
            int s_j = s_have ? ss.j0 : 0;
            bool q_ok = false;
            uint32_t s_g = 0;
            bool o_have = !*abort_flag && it.next(sg);
            int o_j = o_have ? sg.j0 : 0;
            // the issuer polls its barriers without blocking: allow 16 polls per wait poll
            uint32_t idle = 0;
            while (o_have) {
                // ---- O of tile g
                if (g < s_g && ptx::mbar_test(&p_ready[g & 1], (g >> 1) & 1)) {
                    ptx::tc_fence_after();
                    const uint32_t v = ptx::smem_u32(tiles + (g % kStages) * kStride);
                    const bool first = (o_j == sg.j0);
#pragma unroll
                    for (int k = 0; k < kT / 16; ++k)
                        ptx::mma_ts(tmem + kColO, tmem + kColP + 32 * (g & 1) + 8 * k,
                                    ptx::desc_mnmajor_sw128(v + 2048 * k, kChunkBytes), idesc_o, !(first && k == 0));
                    ptx::mma_commit(&o_done[g & 1]);
                    ptx::mma_commit(&tile_empty[g % kStages]);
                    ++g;
                    if (++o_j == sg.j1) {
                        o_have = it.next(sg);
                        o_j = o_have ? sg.j0 : 0;
                    }
                    idle = 0;
                    continue;
                }
                // ---- S of tile s_g
                if (s_have) {
                    const bool first = (s_j == ss.j0);
                    if (first && !q_ok && ptx::mbar_test(q_ready, sidx & 1)) {
                        q_ok = true;
                        ++sidx;
                    }
                    const int st = s_g % kStages;
                    if ((!first || q_ok) && ptx::mbar_test(&tile_full[st], (s_g / kStages) & 1) &&
                        (s_g == 0 || ptx::mbar_test(s_free, (s_g - 1) & 1))) {
                        ptx::tc_fence_after();
                        const uint32_t t = ptx::smem_u32(tiles + st * kStride);
#pragma unroll
                        for (int ks = 0; ks < 16; ++ks)   // latent columns: 4 chunks x 4 K-steps
                            ptx::mma_ts(tmem + kColS, tmem + kColQ + 8 * ks,
                                        ptx::desc_kmajor_sw128(t + (ks >> 2) * kChunkBytes + (ks & 3) * 32), idesc_s,
                                        ks != 0);
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks)    // this CTA's half of the rotary columns
                            ptx::mma_ss(tmem + kColS, ptx::desc_kmajor_sw64(ptx::smem_u32(qrope) + 32 * ks),
                                        ptx::desc_kmajor_sw64(t + 4 * kChunkBytes + 32 * ks), idesc_sr, 1);
                        ptx::mma_commit(s_full);
                        ++s_g;
                        q_ok = false;
                        if (++s_j == ss.j1) {
                            s_have = its.next(ss);
                            s_j = s_have ? ss.j0 : 0;
                        }
                        idle = 0;
                        continue;
                    }
                }
                if (++idle > (ptx::g_wait_limit << 4) || *abort_flag) {
                    ok = false;
                    break;
                }
            }
            if (!ok) fail(err_code, err_detail, abort_flag, 2);
            // drain: wait (bounded) for every MMA issued above before TMEM is released
            ptx::mma_commit(drain);
            if (!ptx::mbar_wait(drain, 0, nullptr)) fail(err_code, err_detail, abort_flag, 4);
        }
    } else {
        // warps 2-5 send partial scores, warps 6-13 run the softmax; warp w works on TMEM
        // lanes 32 * (w % 4) .. +31, so thread h of either role owns head h
        const int sub = warp & 3;
        const int h = sub * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(sub * 32) << 16);
        const bool sender = warp < 6;
        bool ok = true;
        // waits are made warp-uniform so the warp-collective TMEM instructions never diverge
        auto uwait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, abort_flag));
        };
        auto uwait_cluster = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, ptx::mbar_wait_cluster(bar, parity, abort_flag));
        };
        // exchange rows are 128 B (64 bf16); 16-byte chunk v of row h sits at chunk
        // v ^ (h & 7), so a warp's row accesses hit all 32 banks
        Seg cur;
        bool have = it.next(cur);
        int j = have ? cur.j0 : 0;
        uint32_t g = 0;
        if (sender) {
            // ------------------------------------------------------- score senders
            // Q_r of query v: 256 latent columns of this head -> TMEM, 32 rotary columns -> smem
            auto load_q = [&](int v) {
                const uint4* ql = (const uint4*)(q_lat + ((long long)v * 128 + h) * 512 + 256 * rank);
                const uint4* qr = (const uint4*)(q_rope + v * sQr_b + h * sQr_h + 32 * rank);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const uint4 x = ql[c * 8 + v];
                        r[4 * v] = x.x; r[4 * v + 1] = x.y; r[4 * v + 2] = x.z; r[4 * v + 3] = x.w;
                    }
                    ptx::tmem_st32(lane_addr + kColQ + 32 * c, r);
                }
                // rotary part: row h of the shared-memory A operand (64 B, 64-byte swizzle)
#pragma unroll
                for (int v = 0; v < 4; ++v) *(uint4*)(qrope + h * 64 + ((v ^ ((h >> 1) & 3)) << 4)) = qr[v];
                ptx::fence_proxy_async_smem();   // read by the tensor cores
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(q_ready);
            };
            pdl_wait();   // q_lat is written by the previous kernel of this call
            if (have) load_q(cur.v);
            while (have) {
                const uint32_t b = g % kXB, u = g / kXB;
                // partial scores: TMEM -> registers -> bf16 pairs
                if (!uwait(s_full, g & 1)) { ok = false; break; }
                ptx::tc_fence_after();
                uint32_t own[32];
                {
                    uint32_t r[32];
                    float sc[kT];
                    ptx::tmem_ld32(lane_addr + kColS, r);
                    ptx::tmem_ld32x2_second(lane_addr + kColS + 32, sc, r);
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(s_free);
                    // raw partial scores rounded to bf16 pairs (nearest even, in hardware);
                    // both CTAs add the same two rounded partials
#pragma unroll
                    for (int i = 0; i < kT; i += 2) own[i / 2] = ptx::pack_bf16(sc[i], sc[i + 1]);
                }
                // staging buffer b is free once the local softmax read it (tile g - kXB) and
                // the peer read the copy made from it
                if (g >= kXB && !(uwait(&xs_free[b], (u - 1) & 1) && uwait_cluster(&x_empty[b], (u - 1) & 1))) {
                    ok = false;
                    break;
                }
                uint4* row = (uint4*)(xstage + b * kXBytes + h * kXRowBytes);
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    row[v ^ (h & 7)] = make_uint4(own[4 * v], own[4 * v + 1], own[4 * v + 2], own[4 * v + 3]);
                ptx::fence_proxy_async_smem();   // the copy engine reads what this thread wrote
                ptx::mbar_arrive(&xs_ready[b]);
                if (h == 0) {
                    if (!ptx::mbar_wait(&xs_ready[b], u & 1, abort_flag)) {
                        fail(err_code, err_detail, abort_flag, 5);
                    } else {
                        ptx::bulk_copy_to_peer(mapa(ptx::smem_u32(xbuf + b * kXBytes), peer), xstage + b * kXBytes,
                                               kXBytes, mapa(ptx::smem_u32(&x_full[b]), peer));
                    }
                }
                ++g;
                if (++j == cur.j1) {
                    have = it.next(cur);
                    if (have) {
                        j = cur.j0;
                        load_q(cur.v);   // the S of this piece's last tile is already read
                    }
                }
            }
        } else {
            // ----------------------------------------------------- softmax / epilogue
            // two warps per TMEM subpartition: `half` 0 takes tokens 0-31 of a tile, half 1
            // tokens 32-63, of the same 32 heads; they agree on the running max through
            // shared memory, so the P halves they write share one scale per head
            const int half = warp >= 10 ? 1 : 0;
            float m_run = -INFINITY, l_run = 0.f;   // l_run: this half's share of the row sum
            uint32_t pairs = 0;                     // uses of this pair's barrier
            auto pair_exchange = [&](float v) -> float {   // the partner warp's value for head h
                pair_val[(pairs & 1) * 256 + half * 128 + h] = v;
                ptx::mbar_arrive(&pair_bar[sub]);
                if (!uwait(&pair_bar[sub], pairs & 1)) ok = false;
                const float o = pair_val[(pairs & 1) * 256 + (half ^ 1) * 128 + h];
                ++pairs;
                return o;
            };
            while (have) {
                const uint32_t b = g % kXB, u = g / kXB;
                if (h == 0 && half == 0) ptx::mbar_expect_tx(&x_full[b], kXBytes);
                if (!uwait(&xs_ready[b], u & 1)) { ok = false; break; }
                if (!uwait_cluster(&x_full[b], u & 1)) { ok = false; break; }
                // full scores of this half = own + peer partial, both bf16-valued
                float s[kT / 2];
                {
                    const uint4* mine = (const uint4*)(xstage + b * kXBytes + h * kXRowBytes);
                    const uint4* theirs = (const uint4*)(xbuf + b * kXBytes + h * kXRowBytes);
#pragma unroll
                    for (int vv = 0; vv < 4; ++vv) {
                        const int v = 4 * half + vv;
                        const uint4 x = mine[v ^ (h & 7)], y = theirs[v ^ (h & 7)];
                        const uint32_t a4[4] = {x.x, x.y, x.z, x.w};
                        const uint32_t b4[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            s[8 * vv + 2 * q] = __uint_as_float(a4[q] << 16) + __uint_as_float(b4[q] << 16);
                            s[8 * vv + 2 * q + 1] =
                                __uint_as_float(a4[q] & 0xFFFF0000u) + __uint_as_float(b4[q] & 0xFFFF0000u);
                        }
                    }
                    ptx::mbar_arrive(&xs_free[b]);
                    __syncwarp();
                    if (lane == 31) ptx::mbar_arrive_cluster_relaxed(&x_empty[b], peer);
                }
                const bool first = (j == cur.j0);
                if (first) {
                    m_run = -INFINITY;
                    l_run = 0.f;
                }
                // scores are raw dot products here; scale_log2 (softmax scale x log2 e) turns
                // them into base-2 exponents inside one FFMA per probability
                const int valid = min(kT, cur.L - j * kT) - half * (kT / 2);
                if (valid < kT / 2) {   // only a piece's last tile is partial
#pragma unroll
                    for (int i = 0; i < kT / 2; ++i) s[i] = i < valid ? s[i] : -INFINITY;
                }
                float mt = -INFINITY;
#pragma unroll
                for (int i = 0; i < kT / 2; ++i) mt = fmaxf(mt, s[i]);
                mt = fmaxf(mt, pair_exchange(mt));   // tile max over all 64 tokens
                if (!ok) break;
                float alpha = 1.f;
                if (mt * scale_log2 > m_run + kRescaleThreshold) {   // m_run in base-2 units
                    const float m_new = mt * scale_log2;
                    alpha = ex2_ftz(m_run - m_new);
                    m_run = m_new;
                }
                uint32_t pw[kT / 4];
                float sum = 0.f;
#pragma unroll
                for (int i = 0; i < kT / 2; i += 2) {
                    const float p0 = ex2_ftz(fmaf(s[i], scale_log2, -m_run));
                    const float p1 = ex2_ftz(fmaf(s[i + 1], scale_log2, -m_run));
                    sum += p0 + p1;
                    pw[i / 2] = kF8 ? ptx::pack_f16(p0, p1) : ptx::pack_bf16(p0, p1);
                }
                l_run = l_run * alpha + sum;
                const uint32_t pb = g & 1;
                // P buffer pb is free once O of tile g - 2 has completed
                if (g >= 2 && !uwait(&o_done[pb], ((g - 2) >> 1) & 1)) { ok = false; break; }
                ptx::tc_fence_after();
                if (__any_sync(0xffffffffu, !first && alpha != 1.f)) {
                    // O is scaled only once it holds every earlier tile (rare: the running max
                    // moves only when a tile exceeds it by more than the threshold)
                    if (g >= 1 && !uwait(&o_done[(g - 1) & 1], ((g - 1) >> 1) & 1)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const float a = first ? 1.f : alpha;
#pragma unroll 1
                    for (int c0 = 128 * half; c0 < 128 * half + 128; c0 += 32) {
                        uint32_t r[32];
                        ptx::tmem_ld32(lane_addr + kColO + c0, r);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * a);
                        ptx::tmem_st32(lane_addr + kColO + c0, r);
                    }
                }
                ptx::tmem_st16(lane_addr + kColP + 32 * pb + 16 * half, pw);
                const int n_valid = min(kT, cur.L - j * kT);
                if (n_valid < kT) {
                    // The rows past the sequence end in this tile hold whatever follows it
                    // (another sequence, unused capacity, the rest of a page), possibly NaN or
                    // Inf bit patterns, which the O MMA would turn into NaN even with P = 0:
                    // zero them (the score MMA that also read them has completed).
                    uint4* t4 = (uint4*)(tiles + (g % kStages) * kStride);
                    const int tid = (warp - 6) * 32 + lane;   // 0 .. 255 over the softmax warps
                    for (int e = tid; e < (kT - n_valid) * 4 * 8; e += 256) {
                        const int r = n_valid + (e >> 5), c = (e >> 3) & 3, u = e & 7;
                        t4[(c * kChunkBytes + r * 128) / 16 + u] = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();   // read by the tensor cores
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(&p_ready[pb]);
                if (j + 1 == cur.j1) {
                    // piece epilogue: this piece's normalised output O_r / l -> part_o[slot][h][c]
                    // as fp16 (each half writes 128 columns, a thread 64 contiguous bytes of
                    // its head's row at a time); (m, l) from CTA 0
                    const float l_all = l_run + pair_exchange(l_run);
                    if (!ok) break;
                    if (!uwait(&o_done[g & 1], (g >> 1) & 1)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const float inv_l = 1.f / l_all;   // l_all >= 1: the maximum's own p is 1
                    __half* po = part_o + ((long long)cur.slot * 128 + h) * 512 + 256 * rank;
#pragma unroll 1
                    for (int c0 = 128 * half; c0 < 128 * half + 128; c0 += 32) {
                        uint32_t r[32];
                        ptx::tmem_ld32(lane_addr + kColO + c0, r);
                        ptx::tmem_wait_ld();
                        uint32_t hw[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float a = fminf(fmaxf(__uint_as_float(r[2 * j]) * inv_l, -65504.f), 65504.f);
                            const float b = fminf(fmaxf(__uint_as_float(r[2 * j + 1]) * inv_l, -65504.f), 65504.f);
                            hw[j] = ptx::pack_f16(a, b);
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *(uint4*)(po + c0 + 8 * q) = make_uint4(hw[4 * q], hw[4 * q + 1], hw[4 * q + 2], hw[4 * q + 3]);
                    }
                    if (rank == 0 && half == 0) {
                        part_ml[((long long)cur.slot * 128 + h) * 2] = m_run;
                        part_ml[((long long)cur.slot * 128 + h) * 2 + 1] = l_all;
                    }
                    ptx::tc_fence_before();
                }
                ++g;
                if (++j == cur.j1) {
                    have = it.next(cur);
                    j = have ? cur.j0 : 0;
                }
            }
        }
        if (!ok) fail(err_code, err_detail, abort_flag, 3);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
    cluster_sync_all();  // neither CTA leaves while its peer may still touch its shared memory
}

// ------------------------------------------------------------- merge + W_UV
// o[v,h,:] = W_UV[h] o_lat[v,h,:],  o_lat[v,h,c] = sum_p 2^(m_p - M) l_p Ob_p[h,c] / sum_p 2^(m_p - M) l_p
// over the pieces p of query v, Ob_p = O_p / l_p being piece p's normalised output (fp16)
// (M = max_p m_p; a query with no row gives o = 0); query v is query v % Q of sequence
// v / Q.  One CTA per (head h, block of BN queries).  Thread 0 starts the bulk loads of the
// tiled W_UV[h] (128 x 512 fp16, the A operand) before waiting for the decode kernel; the
// sixteen warps then merge the partials of their rows (lane per 16 columns, two rows per
// load round) straight into the B operand in shared memory as fp16 (K-major, 128-byte
// swizzle, as TMA would lay it out); one thread issues the 32 MMAs (M = 128, N = BN, fp16
// operands, fp32 accumulation) and four warps store D = o[:, h, :]^T as bf16.  fp16 keeps
// o_lat's rounding at 2^-12 (bf16 would add 2^-9 after the partials' own fp16 rounding).
constexpr int kMergeThreads = 512;
constexpr int kMergeABytes = 8 * 128 * 128;   // W_UV[h]: 8 chunks of 128 rows x 64 columns

template <int BN>
constexpr int merge_smem() { return kMergeABytes + 8 * BN * 128 + 1024 + 64; }

// kLat: the merged, normalised o_lat rows themselves are the output (fp16, saturated, at
// o[v, h, :] with strides sO_b, sO_h): no W_UV product (the folded weights apply W_UV inside
// W_O, whose product takes o_lat in fp16).
template <int BN, bool kSib, bool kLat = false>
__global__ void __launch_bounds__(kMergeThreads, 1)
merge_wuv_kernel(const __nv_bfloat16* __restrict__ uv, const SeqSrc src, int P, int B, int Q_arg,
                 const __half* __restrict__ part_o, const float* __restrict__ part_ml, __nv_bfloat16* __restrict__ o,
                 long long sO_b, long long sO_h, int* err_code, long long* err_detail) {
    extern __shared__ uint8_t merge_smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)merge_smem_raw + 1023) & ~(uintptr_t)1023);
    const int Q = kSib ? Q_arg : 1;   // queries per sequence
    uint8_t* sA = smem;
    uint8_t* sB = smem + kMergeABytes;
    uint64_t* a_full = (uint64_t*)(sB + 8 * BN * 128);
    uint64_t* d_full = a_full + 1;
    uint32_t* tmem_slot = (uint32_t*)(d_full + 1);
    const int h = blockIdx.x, n0 = blockIdx.y * BN;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        ptx::mbar_init(a_full, 1);
        ptx::mbar_init(d_full, 1);
        ptx::fence_mbar_init();
        if (!kLat) {
            // the weights are not written by earlier kernels: load them before waiting; the
            // tiled copy is already the shared-memory image, 8 contiguous 16 KB chunks per head
            ptx::mbar_expect_tx(a_full, kMergeABytes);
            const uint8_t* src = (const uint8_t*)uv + (size_t)h * kMergeABytes;
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) ptx::bulk_load(sA + kc * 16384, src + kc * 16384, 16384, a_full);
        }
    }
    if (!kLat && warp == 1) {
        ptx::tmem_alloc(tmem_slot, BN);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) pdl_trigger();
    // The split of the decode kernel (same cost model, same cluster count, same sibling
    // groups), recomputed from the sequence lengths before waiting for that kernel: cost
    // positions of the first and one past the last tile of this CTA's queries.
    __shared__ int s_wsum[kMergeThreads / 32];
    __shared__ int s_pos[2][BN];
    constexpr int kW = kMergeThreads / 32;
    int total = 0;
    {
        int mine = 0;
        for (int b = threadIdx.x; b < B; b += kMergeThreads) mine += cost_of_tiles(tiles_of_len(src.len(b)));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
        if (lane == 0) s_wsum[warp] = mine;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kW; ++i) total += s_wsum[i];
        __syncthreads();
    }
    const int R = P / Q;
    const int per = total > 0 ? (total + R - 1) / R : 1;
    const int NV = B * Q;   // queries
    {
        int carry = 0;
        for (int c0 = 0; c0 < B && c0 * Q < n0 + BN; c0 += kMergeThreads) {
            const int b = c0 + (int)threadIdx.x;
            const int nt = b < B ? tiles_of_len(src.len(b)) : 0;
            const int cb = cost_of_tiles(nt);
            int incl = cb;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            if (lane == 31) s_wsum[warp] = incl;
            __syncthreads();
            int before = carry, chunk = 0;
#pragma unroll
            for (int i = 0; i < kW; ++i) {
                const int v = s_wsum[i];
                before += i < warp ? v : 0;
                chunk += v;
            }
            const int cs = before + incl - cb;
            if (!kSib) {
                if (b < B && b >= n0 && b < n0 + BN) {
                    s_pos[0][b - n0] = cs + kPieceCost;
                    s_pos[1][b - n0] = cs + kPieceCost + nt;
                }
            } else if (b < B) {
                const int Lb = nt > 0 ? src.len(b) : 0;
                for (int t = 0; t < Q; ++t) {
                    const int v = b * Q + t;
                    if (v >= n0 && v < n0 + BN) {
                        const int ntt = tiles_of_len(Lb - (Q - 1 - t));
                        s_pos[0][v - n0] = ntt > 0 ? cs + kPieceCost : 0;
                        s_pos[1][v - n0] = ntt > 0 ? cs + kPieceCost + ntt : 0;
                    }
                }
            }
            carry += chunk;
            __syncthreads();
        }
    }
    pdl_wait();   // the partials come from the decode kernel

    constexpr int kRowsPerWarp = BN / kW;
    // rows merged per load round: the requests of kRound rows are in flight together
    constexpr int kRound = kRowsPerWarp < 2 ? kRowsPerWarp : 2;
    int t0r[kRowsPerWarp], t1r[kRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int v = n0 + warp + kW * i;
        t0r[i] = v < NV ? s_pos[0][warp + kW * i] : 0;
        t1r[i] = v < NV ? s_pos[1][warp + kW * i] : 0;
    }
    // Piece p of a row holds its normalised partial O_p / l_p (fp16, 16 columns per lane)
    // and (m_p, l_p); piece 0 (from range t0 / per) is in slot v, piece p > 0 continues the
    // query in range t0 / per + p, i.e. in sibling cluster (t0 / per + p) Q + tq, and is in
    // slot NV + that cluster.  The weight of piece p is 2^(m_p - M) l_p.
#pragma unroll 1
    for (int i0 = 0; i0 < kRowsPerWarp; i0 += kRound) {
        float2 ml[kRound];
        uint4 x[kRound][4][2];
        int np[kRound], cfirst[kRound];
        long long slot_base[kRound] = {};   // slot of piece p > 0: slot_base + p * Q
        auto slot_of = [&](int k, int p) -> long long {
            return p == 0 ? (long long)(n0 + warp + kW * (i0 + k)) : slot_base[k] + (long long)p * Q;
        };
        // requests of every row of the round: (m, l) of up to 32 pieces (lane p) and the
        // first four pieces' partial rows
#pragma unroll
        for (int k = 0; k < kRound; ++k) {
            const int i = i0 + k, v = n0 + warp + kW * i, tq = kSib ? v % Q : 0;
            const int t0 = t0r[i], t1 = t1r[i];
            cfirst[k] = t1 > t0 ? t0 / per : 0;
            np[k] = t1 > t0 ? (t1 - 1) / per - cfirst[k] + 1 : 0;
            slot_base[k] = kSib ? NV + (long long)cfirst[k] * Q + tq : (long long)B + cfirst[k];
            ml[k] = lane < np[k] ? *(const float2*)(part_ml + (slot_of(k, lane) * 128 + h) * 2)
                                 : make_float2(-INFINITY, 0.f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4* src =
                    (const uint4*)(part_o + (slot_of(k, q < np[k] ? q : 0) * 128 + h) * 512 + 16 * lane);
                x[k][q][0] = q < np[k] ? src[0] : make_uint4(0, 0, 0, 0);
                x[k][q][1] = q < np[k] ? src[1] : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int k = 0; k < kRound; ++k) {
            const int r = warp + kW * (i0 + k);
            float acc[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[c] = 0.f;
            if (np[k] > 0) {
                float M = ml[k].x;
                for (int p = 32 + lane; p < np[k]; p += 32) M = fmaxf(M, part_ml[(slot_of(k, p) * 128 + h) * 2]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
                const float w_lane = lane < np[k] ? exp2f(ml[k].x - M) * ml[k].y : 0.f;
                float L = w_lane;
                for (int p = 32 + lane; p < np[k]; p += 32) {
                    const float2 v2 = *(const float2*)(part_ml + (slot_of(k, p) * 128 + h) * 2);
                    L += exp2f(v2.x - M) * v2.y;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
                for (int p0 = 0;; p0 += 4) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int p = p0 + q;
                        float w = __shfl_sync(0xffffffffu, w_lane, p & 31);
                        if (p >= 32 && p < np[k]) {
                            const float2 v2 = *(const float2*)(part_ml + (slot_of(k, p) * 128 + h) * 2);
                            w = exp2f(v2.x - M) * v2.y;
                        }
                        if (p >= np[k]) w = 0.f;
#pragma unroll
                        for (int hv = 0; hv < 2; ++hv) {
                            const uint32_t wd[4] = {x[k][q][hv].x, x[k][q][hv].y, x[k][q][hv].z, x[k][q][hv].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wd[e]));
                                acc[8 * hv + 2 * e] = fmaf(w, f.x, acc[8 * hv + 2 * e]);
                                acc[8 * hv + 2 * e + 1] = fmaf(w, f.y, acc[8 * hv + 2 * e + 1]);
                            }
                        }
                    }
                    if (p0 + 4 >= np[k]) break;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {   // the next four pieces
                        const int p = p0 + 4 + q;
                        const uint4* src =
                            (const uint4*)(part_o + (slot_of(k, p < np[k] ? p : 0) * 128 + h) * 512 + 16 * lane);
                        x[k][q][0] = p < np[k] ? src[0] : make_uint4(0, 0, 0, 0);
                        x[k][q][1] = p < np[k] ? src[1] : make_uint4(0, 0, 0, 0);
                    }
                }
                const float inv = 1.f / L;
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[c] *= inv;
            }
            if (kLat) {   // o_lat[v, h, 16 lane ..] as fp16 (saturated), one rounding
                const int v = n0 + r;
                if (v < NV) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) acc[c] = fminf(fmaxf(acc[c], -65504.f), 65504.f);
                    uint4* dst = (uint4*)(o + v * sO_b + h * sO_h + 16 * lane);
#pragma unroll
                    for (int hv = 0; hv < 2; ++hv)
                        dst[hv] = make_uint4(ptx::pack_f16(acc[8 * hv], acc[8 * hv + 1]),
                                             ptx::pack_f16(acc[8 * hv + 2], acc[8 * hv + 3]),
                                             ptx::pack_f16(acc[8 * hv + 4], acc[8 * hv + 5]),
                                             ptx::pack_f16(acc[8 * hv + 6], acc[8 * hv + 7]));
                }
                continue;
            }
            // o_lat as fp16 (saturated), the B operand of the W_UV product: columns 16 lane ..
            // +15 = chunk lane / 4, 16-byte units 2 (lane % 4) and +1 of row r
            uint8_t* rowp = sB + (lane >> 2) * (BN * 128) + r * 128;
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[c] = fminf(fmaxf(acc[c], -65504.f), 65504.f);
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
                const int u = 2 * (lane & 3) + hv;
                *(uint4*)(rowp + ((u ^ (r & 7)) << 4)) =
                    make_uint4(ptx::pack_f16(acc[8 * hv], acc[8 * hv + 1]), ptx::pack_f16(acc[8 * hv + 2], acc[8 * hv + 3]),
                               ptx::pack_f16(acc[8 * hv + 4], acc[8 * hv + 5]),
                               ptx::pack_f16(acc[8 * hv + 6], acc[8 * hv + 7]));
            }
        }
    }
    if (kLat) return;   // no W_UV product, no TMEM
    ptx::fence_proxy_async_smem();   // the tensor cores read what the threads wrote
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    if (threadIdx.x == 32) {
        if (!ptx::mbar_wait(a_full, 0, nullptr)) {
            latch(DevErr{err_code, err_detail}, kErrTimeout, 8000000 + h);
            ok = false;
        } else {
            ptx::tc_fence_after();
            // A = W_UV[h] and B = o_lat, both fp16
            constexpr uint32_t idesc = ptx::idesc_f16_f32(128, BN, 0, 0);
#pragma unroll
            for (int kc = 0; kc < 8; ++kc)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    ptx::mma_ss(tmem, ptx::desc_kmajor_sw128(ptx::smem_u32(sA + kc * 16384) + 32 * k),
                                ptx::desc_kmajor_sw128(ptx::smem_u32(sB + kc * BN * 128) + 32 * k), idesc,
                                (kc | k) != 0);
        }
        ptx::mma_commit(d_full);   // also after a timeout: nothing issued, completes at once
    }
    if (warp < 4) {
        if (!ptx::mbar_wait(d_full, 0, nullptr)) {
            if (lane == 0) latch(DevErr{err_code, err_detail}, kErrTimeout, 8100000 + h);
        } else {
            ptx::tc_fence_after();
            // D (row m = TMEM lane, column = sequence) -> bf16 stage[b][m] in the A buffer
            // (free once the MMAs completed), then whole 256-byte rows o[b, h, :]
            const int m = warp * 32 + lane;
            __nv_bfloat16* stage = (__nv_bfloat16*)sA;
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t r[32];
                ptx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) stage[(c0 + j) * 128 + m] = __float2bfloat16_rn(__uint_as_float(r[j]));
            }
        }
        ptx::named_barrier_sync(1, 128);   // the four epilogue warps
        for (int i = threadIdx.x; i < BN * 16; i += 128) {
            const int v = n0 + (i >> 4);
            if (v < NV) ((uint4*)(o + v * sO_b + h * sO_h))[i & 15] = ((const uint4*)sA)[i];
        }
    }
    (void)ok;
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, BN);
}

// ------------------------------------------------------------- weight tiling
// One thread per 16-byte unit of the tiled copies: unit u of row r of chunk c of head h goes
// to unit u ^ (r % 8) of that row (the 128-byte swizzle of a 1024-byte-aligned operand).
__global__ void __launch_bounds__(256)
tile_weights_kernel(const __nv_bfloat16* __restrict__ W_UKT, const __nv_bfloat16* __restrict__ W_UV,
                    __nv_bfloat16* __restrict__ ukt, __nv_bfloat16* __restrict__ uv) {
    const long long n = (long long)kH * 8 * 128 * 8;   // units per tensor
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < 2 * n; i += (long long)gridDim.x * blockDim.x) {
        const bool is_uv = i >= n;
        const long long k = is_uv ? i - n : i;
        const int u = (int)(k & 7), r = (int)((k >> 3) & 127), c = (int)((k >> 10) & 7), h = (int)(k >> 13);
        const uint4* src;
        if (!is_uv)   // chunk c = 2t + kk: W_UK^T[h][128t + r][64kk + 8u ..]
            src = (const uint4*)(W_UKT + ((long long)h * kDc + 128 * (c >> 1) + r) * 128 + 64 * (c & 1) + 8 * u);
        else          // chunk c: W_UV[h][r][64c + 8u ..]
            src = (const uint4*)(W_UV + ((long long)h * 128 + r) * kDc + 64 * c + 8 * u);
        uint4* dst = (uint4*)((is_uv ? uv : ukt) + (((long long)h * 8 + c) * 128 + r) * 64) + (u ^ (r & 7));
        uint4 x = *src;
        if (is_uv) {   // W_UV in fp16 (the merge's product runs on fp16 operands)
            uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
                w[q] = ptx::pack_f16(fminf(fmaxf(lo, -65504.f), 65504.f), fminf(fmaxf(hi, -65504.f), 65504.f));
            }
            x = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *dst = x;
    }
}

// Kernel attributes, set once per kernel: the dynamic shared memory it needs, and the
// largest shared-memory carve-out for every kernel of the chain, so that consecutive kernels
// find the SMs already configured.
template <typename K>
cudaError_t set_smem_attrs(K kernel, int bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    return e;
}

// ----------------------------------------------------------------- q absorption
// q_lat[b,h,:] = W_UK[h]^T q_nope[b,h,:], as D[512 x BN] = W_UK^T[h] (512 x 128) . Q_h^T with
// Q_h = q_nope[n0 .. n0+BN, h, :].  One CTA per (head, block of BN sequences) holds the whole
// W_UK^T[h] (8 contiguous 16 KB chunks of the tiled copy, 128 KB) and Q_h (2 TMA boxes), issues 4 x 8 MMAs into four
// BN-column TMEM accumulators (one per 128-row tile) and stores q_lat.
// This is the first kernel of the decode chain: it waits for all earlier work before it lets
// the next kernel launch (the decode kernel then reads the cache without waiting).
constexpr int kAbsorbThreads = 128;
constexpr int kAbsorbTiles = 2;   // 128-row tiles of W_UK^T[h] per CTA (two CTAs per head)

template <int BN>
constexpr int absorb_smem() { return 2 * kAbsorbTiles * 16384 + 2 * BN * 128 + 1024 + 64; }

// q_lat is stored as bf16, or (kF16) as fp16 saturated to +-65504 for the FP8-row decode,
// whose latent MMAs run on fp16 operands.
template <int BN, bool kF16>
__global__ void __launch_bounds__(kAbsorbThreads, 1)
absorb_q_kernel(const __nv_bfloat16* __restrict__ ukt, const __grid_constant__ CUtensorMap tm_q, int B,
                __nv_bfloat16* __restrict__ q_lat, int* err_code, long long* err_detail) {
    extern __shared__ uint8_t absorb_smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)absorb_smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sA = smem;                                 // [m tile][k chunk] chunks of 128 rows x 128 B
    uint8_t* sB = smem + 2 * kAbsorbTiles * 16384;      // [k chunk] boxes of BN rows x 128 B
    uint64_t* full = (uint64_t*)(sB + 2 * BN * 128);
    uint64_t* d_full = full + 1;
    uint32_t* tmem_slot = (uint32_t*)(d_full + 1);
    constexpr int W = 128 * kAbsorbTiles;   // latent columns of q_lat this CTA writes
    const int h = blockIdx.x / (4 / kAbsorbTiles), t0 = (blockIdx.x % (4 / kAbsorbTiles)) * kAbsorbTiles;
    const int n0 = blockIdx.y * BN;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        ptx::mbar_init(full, 1);
        ptx::mbar_init(d_full, 1);
        ptx::fence_mbar_init();
        ptx::tma_prefetch(&tm_q);
        ptx::mbar_expect_tx(full, 2 * kAbsorbTiles * 16384 + 2 * BN * 128);
        // weights first (earlier kernels do not write them): the tiled copy is already the
        // shared-memory image, chunk (t, k) at (2t + k) x 16 KB; this CTA takes tiles t0 ..
        const uint8_t* src = (const uint8_t*)ukt + ((size_t)h * 8 + 2 * t0) * 16384;
#pragma unroll
        for (int c = 0; c < 2 * kAbsorbTiles; ++c) ptx::bulk_load(sA + c * 16384, src + c * 16384, 16384, full);
        pdl_wait();      // the queries may come from the previous kernel; all earlier work is done
        pdl_trigger();   // only now may the next kernel launch
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) ptx::tma_load_3d(sB + kc * BN * 128, &tm_q, full, 64 * kc, n0, h);
    }
    constexpr uint32_t kCols = kAbsorbTiles * BN < 32 ? 32 : kAbsorbTiles * BN;
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, kCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 32) {
        if (!ptx::mbar_wait(full, 0, nullptr)) {
            latch(DevErr{err_code, err_detail}, kErrTimeout, 8200000 + h);
        } else {
            ptx::tc_fence_after();
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, BN, 0, 0);
#pragma unroll
            for (int mt = 0; mt < kAbsorbTiles; ++mt)
#pragma unroll
                for (int kc = 0; kc < 2; ++kc)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        ptx::mma_ss(tmem + mt * BN, ptx::desc_kmajor_sw128(ptx::smem_u32(sA + (mt * 2 + kc) * 16384) + 32 * k),
                                    ptx::desc_kmajor_sw128(ptx::smem_u32(sB + kc * BN * 128) + 32 * k), idesc,
                                    (kc | k) != 0);
        }
        ptx::mma_commit(d_full);   // after a timeout nothing was issued and this completes at once
    }
    if (!ptx::mbar_wait(d_full, 0, nullptr)) {
        if (lane == 0) latch(DevErr{err_code, err_detail}, kErrTimeout, 8300000 + h);
    } else {
        ptx::tc_fence_after();
        // D (row = latent index, column = sequence) -> bf16 stage[b][128 x kAbsorbTiles] in the
        // A buffer (free once the MMAs completed), then whole rows of q_lat[b, h, 128 t0 ..]
        const int m = warp * 32 + lane;   // row of the 128-row tile = TMEM lane
        __nv_bfloat16* stage = (__nv_bfloat16*)sA;
#pragma unroll 1
        for (int mt = 0; mt < kAbsorbTiles; ++mt)
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t r[32];
                ptx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + mt * BN + c0, r);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float x = __uint_as_float(r[j]);
                    stage[(c0 + j) * W + 128 * mt + m] =
                        kF16 ? __ushort_as_bfloat16(__half_as_ushort(__float2half_rn(fminf(fmaxf(x, -65504.f), 65504.f))))
                             : __float2bfloat16_rn(x);
                }
            }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < BN * (W / 8); i += kAbsorbThreads) {
        const int b = n0 + i / (W / 8);
        if (b < B) ((uint4*)(q_lat + ((long long)b * 128 + h) * 512 + 128 * t0))[i % (W / 8)] = ((const uint4*)sA)[i];
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) ptx::tmem_dealloc(tmem, kCols);
}

template <int BN, bool kF16>
cudaError_t launch_absorb(const __nv_bfloat16* ukt, const CUtensorMap& mq, int B, __nv_bfloat16* q_lat, int* err_code,
                          long long* err_detail, cudaStream_t s) {
    static const cudaError_t attr = set_smem_attrs(absorb_q_kernel<BN, kF16>, absorb_smem<BN>());
    if (attr != cudaSuccess) return attr;
    return launch_pdl(absorb_q_kernel<BN, kF16>, dim3(128 * (4 / kAbsorbTiles), (B + BN - 1) / BN),
                      dim3(kAbsorbThreads), absorb_smem<BN>(), s, ukt, mq, B, q_lat, err_code, err_detail);
}

template <bool kF16>
cudaError_t launch_absorb_any(int NV, const __nv_bfloat16* ukt, const CUtensorMap& mq, __nv_bfloat16* q_lat,
                              int* err_code, long long* err_detail, cudaStream_t s) {
    return NV <= 32   ? launch_absorb<32, kF16>(ukt, mq, NV, q_lat, err_code, err_detail, s)
           : NV <= 64 ? launch_absorb<64, kF16>(ukt, mq, NV, q_lat, err_code, err_detail, s)
                      : launch_absorb<128, kF16>(ukt, mq, NV, q_lat, err_code, err_detail, s);
}

template <bool kSib, bool kLat = false>
cudaError_t launch_merge(int NV, const __nv_bfloat16* uv, const SeqSrc& seqs, int P, int B, int Q, const DecodeWs& ws,
                         __nv_bfloat16* o, int* err_code, long long* err_detail, cudaStream_t s) {
    // o [NV, 128 heads, 128] (W_UV applied), or o_lat [NV, 128 heads, 512] (kLat)
    const long long sO_b = kLat ? 128LL * 512 : 128LL * 128, sO_h = kLat ? 512 : 128;
    if (NV <= 32) {
        static const cudaError_t attr = set_smem_attrs(merge_wuv_kernel<32, kSib, kLat>, merge_smem<32>());
        if (attr != cudaSuccess) return attr;
        return launch_pdl(merge_wuv_kernel<32, kSib, kLat>, dim3(128, 1), dim3(kMergeThreads), merge_smem<32>(), s,
                          uv, seqs, P, B, Q, (const __half*)ws.part_o, (const float*)ws.part_ml, o, sO_b, sO_h,
                          err_code, err_detail);
    }
    static const cudaError_t attr = set_smem_attrs(merge_wuv_kernel<64, kSib, kLat>, merge_smem<64>());
    if (attr != cudaSuccess) return attr;
    return launch_pdl(merge_wuv_kernel<64, kSib, kLat>, dim3(128, (NV + 63) / 64), dim3(kMergeThreads),
                      merge_smem<64>(), s, uv, seqs, P, B, Q, (const __half*)ws.part_o, (const float*)ws.part_ml, o,
                      sO_b, sO_h, err_code, err_detail);
}

int g_clusters_cached = 0;

template <bool kF8>
int resident_clusters(int num_sms) {
    set_smem_attrs(decode_tc_kernel<kF8, false>, dec_smem<kF8>());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(DecCfg<kF8>::kThreads, 1, 1);
    cfg.dynamicSmemBytes = dec_smem<kF8>();
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_tc_kernel<kF8, false>, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms / 2;
    }
    return n;
}

// Clusters of one decode launch: all resident at once, for both cache formats (the merge
// kernel and the workspace size depend on this count only).
int max_clusters(int num_sms) {
    if (g_clusters_cached > 0) return g_clusters_cached;
    const int a = resident_clusters<false>(num_sms), b = resident_clusters<true>(num_sms);
    g_clusters_cached = a < b ? a : b;
    return g_clusters_cached;
}

}  // namespace

int decode_clusters(int num_sms) { return max_clusters(num_sms); }

cudaError_t set_wait_limit_decode(uint32_t polls) { return ptx::set_wait_limit_of_this_file(polls); }

cudaError_t tile_weights_tc(const __nv_bfloat16* W_UKT, const __nv_bfloat16* W_UV, __nv_bfloat16* ukt,
                            __nv_bfloat16* uv, cudaStream_t s) {
    tile_weights_kernel<<<1184, 256, 0, s>>>(W_UKT, W_UV, ukt, uv);
    return cudaGetLastError();
}

size_t decode_ws_bytes(int B, int num_sms) {
    const size_t P = (size_t)(num_sms / 2);
    const size_t slots = (size_t)B + P + 1;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return up((size_t)B * 128 * 512 * 2) + up(slots * 512 * 128 * 2) + up(slots * 128 * 2 * 4);
}

DecodeWs carve_decode_ws(char* base, int B, int num_sms) {
    const size_t P = (size_t)(num_sms / 2);
    const size_t slots = (size_t)B + P + 1;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    DecodeWs w{};
    size_t off = 0;
    auto take = [&](size_t bytes) -> char* {
        char* p = base ? base + off : nullptr;
        off += up(bytes);
        return p;
    };
    w.q_lat = (__nv_bfloat16*)take((size_t)B * 128 * 512 * 2);
    w.part_o = (__half*)take(slots * 512 * 128 * 2);
    w.part_ml = (float*)take(slots * 128 * 2 * 4);
    w.max_parts = (int)slots;
    return w;
}

cudaError_t decode_absorbed_tc(const __nv_bfloat16* qn, long long sQn_b, long long sQn_h, const __nv_bfloat16* qr,
                               long long sQr_b, long long sQr_h, const __nv_bfloat16* ukt,
                               const __nv_bfloat16* uv, const void* cache, bool fp8, long long cache_rows,
                               const int32_t* offsets, const int32_t* seq_lens, const int32_t* block_table,
                               int bt_stride, int B, int Q, bool stream_once, float scale, __nv_bfloat16* o, const DecodeWs& ws,
                               int num_sms,
                               int* err_code, long long* err_detail, cudaStream_t s, bool folded) {
    if (B <= 0) return cudaSuccess;
    cudaError_t e;
    if (cache_rows <= 0 || cache_rows > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    if (block_table && (!seq_lens || bt_stride <= 0)) return cudaErrorInvalidValue;
    const SeqSrc seqs{offsets, seq_lens, block_table, bt_stride, cache_rows};
    const int P = max_clusters(num_sms);
    if (Q < 1 || Q > P) return cudaErrorInvalidValue;
    const int NV = B * Q;   // queries
    if (!folded) {
        // q_lat[v,h,:] = W_UK[h]^T q_nope[v,h,:]
        ProfScope ps(s, "tc_q_absorb");
        CUtensorMap mq;
        const int BN = NV <= 32 ? 32 : NV <= 64 ? 64 : 128;
        const uint64_t dq[3] = {128, (uint64_t)NV, 128};
        const uint64_t sq[2] = {(uint64_t)sQn_b * 2, (uint64_t)sQn_h * 2};
        const uint32_t bq[3] = {64, (uint32_t)BN, 1};
        if (!make_tmap_bf16(&mq, qn, 3, dq, sq, bq)) return cudaErrorInvalidValue;
        e = fp8 ? launch_absorb_any<true>(NV, ukt, mq, ws.q_lat, err_code, err_detail, s)
                : launch_absorb_any<false>(NV, ukt, mq, ws.q_lat, err_code, err_detail, s);
        if (e != cudaSuccess) return e;
    }
    {
        ProfScope ps(s, fp8 ? "tc_flash_decode_fp8" : "tc_flash_decode");
        CUtensorMap m, mr, msc;
        const float scale_log2 = scale * 1.4426950408889634f;
        if (!fp8) {
            const uint64_t dims[2] = {576, (uint64_t)cache_rows};
            const uint64_t strides[1] = {576 * 2};
            const uint32_t box[2] = {64, (uint32_t)kT};
            const uint32_t box_rope[2] = {32, (uint32_t)kT};
            if (!make_tmap_bf16(&m, cache, 2, dims, strides, box) ||
                !make_tmap_bf16(&mr, cache, 2, dims, strides, box_rope, 64))
                return cudaErrorInvalidValue;
            msc = mr;   // unused
            static const cudaError_t attr1 = set_smem_attrs(decode_tc_kernel<false, false>, dec_smem<false>());
            static const cudaError_t attr2 = set_smem_attrs(decode_tc_kernel<false, true>, dec_smem<false>());
            if (attr1 != cudaSuccess) return attr1;
            if (attr2 != cudaSuccess) return attr2;
            e = launch_pdl(Q > 1 ? decode_tc_kernel<false, true> : decode_tc_kernel<false, false>, dim3(2 * P),
                           dim3(DecCfg<false>::kThreads), dec_smem<false>(), s, m, mr, msc, ws.q_lat, qr, sQr_b, sQr_h,
                           seqs, B, Q, (int)(stream_once ? 1 : 0), (long long)cache_rows, scale_log2, ws.part_o,
                           ws.part_ml, folded ? nullptr : (const uint8_t*)uv, folded ? 0LL : (long long)kTiledWeightBytes,
                           err_code, err_detail);
        } else {
            // FP8 rows of kF8RowBytes: codes as bytes, the rotary key as bf16 elements, the
            // scale field as fp32 elements
            const uint64_t sr[1] = {(uint64_t)kF8RowBytes};
            const uint64_t dc[2] = {(uint64_t)kF8RowBytes, (uint64_t)cache_rows};
            const uint32_t bc[2] = {128, (uint32_t)kT};
            const uint64_t dr[2] = {(uint64_t)kF8RowBytes / 2, (uint64_t)cache_rows};
            const uint32_t br[2] = {32, (uint32_t)kT};
            const uint64_t ds[2] = {(uint64_t)kF8RowBytes / 4, (uint64_t)cache_rows};
            const uint32_t bs[2] = {4, (uint32_t)kT};
            if (!make_tmap(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache, 2, dc, sr, bc, 128) ||
                !make_tmap(&mr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cache, 2, dr, sr, br, 64) ||
                !make_tmap(&msc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cache, 2, ds, sr, bs, 0))
                return cudaErrorInvalidValue;
            if (Q != 1) return cudaErrorInvalidValue;   // FP8 rows: one query per sequence
            static const cudaError_t attr = set_smem_attrs(decode_tc_kernel<true, false>, dec_smem<true>());
            if (attr != cudaSuccess) return attr;
            e = launch_pdl(decode_tc_kernel<true, false>, dim3(2 * P), dim3(DecCfg<true>::kThreads), dec_smem<true>(), s,
                           m, mr, msc, ws.q_lat, qr, sQr_b, sQr_h, seqs, B, Q, (int)(stream_once ? 1 : 0),
                           (long long)cache_rows, scale_log2, ws.part_o, ws.part_ml, (const uint8_t*)uv,
                           (long long)kTiledWeightBytes, err_code, err_detail);
        }
        if (e != cudaSuccess) return e;
    }
    if (folded) {
        // merge of the pieces alone: o = o_lat (W_UV is inside the folded W_O)
        ProfScope ps(s, "tc_merge");
        e = Q > 1 ? launch_merge<true, true>(NV, uv, seqs, P, B, Q, ws, o, err_code, err_detail, s)
                  : launch_merge<false, true>(NV, uv, seqs, P, B, Q, ws, o, err_code, err_detail, s);
    } else {
        // merge of the pieces fused with o[v,h,:] = W_UV[h] o_lat[v,h,:]
        ProfScope ps(s, "tc_merge_w_uv");
        e = Q > 1 ? launch_merge<true>(NV, uv, seqs, P, B, Q, ws, o, err_code, err_detail, s)
                  : launch_merge<false>(NV, uv, seqs, P, B, Q, ws, o, err_code, err_detail, s);
    }
    return e;
}

}  // namespace tc
}  // namespace mla
