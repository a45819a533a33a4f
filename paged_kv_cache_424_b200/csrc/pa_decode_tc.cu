// pa_decode_tc.cu -- paged decode attention for GQA groups (4, 8 or 16 query
// heads per KV head, head_dim 128) on the 5th-generation tensor cores.
//
// Method: "vLLM PagedAttention 大模型推理架构深度实战" section 2.2 (16-token
// blocks reached through the block table) and section 5.1 (exact attention,
// tiles combined by online softmax).  With a query group of G heads sharing
// one KV head, a chunk of 128 cached tokens gives two real dense products:
//   S (128 tokens x 16)  = K (128 x 128 dims) . Q^T (128 x 16)     [QK^T]
//   O^T (128 dims x 16)  = V^T (128 x 128 tokens) . P^T (128 x 16)  [PV]
// (the G query rows padded to the MMA's N = 16).
//
// CTA = (partition, KV head, sequence), or a group of consecutive
// partitions or of two KV heads (set by the host): 8 warps (12 with 16
// columns, whose softmax work is split over 8 warps, 8 columns each); the
// last warp idles.
//   warp 4  K producer and warp 6  V producer (8 and 10 with 16 columns): per chunk, 2-D tiled TMA loads
//           of the 8 blocks' K (or V) rows (16 rows x 64 dims per box,
//           128-byte swizzle) into the K (or V) tile, as soon as the previous
//           chunk's MMA that read the tile has completed; blocks past the
//           partition are loaded from an out-of-range row, which the TMA
//           fills with zeros.  The partition's table slice is read once, 32
//           entries per coalesced load.
//   warp 5  MMA issuer (warp 9 with 16 columns; one thread): S into TMEM (double-buffered), then
//           O = V^T P^T into TMEM (double-buffered), each completion signalled
//           by tcgen05.commit on an mbarrier; allocates / frees TMEM.
//   warps 0-3 softmax: thread t owns TMEM lane t = token t of S and output
//           dim t of O (with 16 columns warps 0-7: warps w and w + 4 share
//           lane quadrant w and take columns 0-7 and 8-15).  Masks tokens past the context, keeps the online
//           softmax with a lazy running max (raised only when some logit
//           beats it by 2^8; a CTA-wide flag skips the max reduction in all
//           other chunks), writes P (same 16-bit type as V) into a swizzled
//           tile, and accumulates O chunk by chunk in registers.
// Shared memory: K tile 32 KiB + V tile 32 KiB + Q 4 KiB + P 4 KiB (+ <1 KiB)
// = 74 KiB, three CTAs per SM; TMEM: 64 columns per CTA.  With 16 columns
// (two CTAs per SM) a second V stage (+32 KiB) lets the V load of the next
// chunk overlap the current chunk's softmax and PV product.
// FP8 E4M3 caches: a chunk's codes take 16 KiB (128-byte swizzle), so each
// 32 KiB tile area holds two stages and the loads of chunk c + 1 overlap the
// products of chunk c.  Both products run E4M3 x E4M3 on the codes as
// loaded: S = K . Q^T against Q split into three E4M3 parts (3G columns,
// rounded up to 16), O^T = V^T . P^T against P split into four (4G
// columns); 64, 128 or 256 TMEM columns for G = 4, 8, 16.
// Results go to `out` (one partition) or to the split workspace for the
// log-sum-exp merge, exactly like the CUDA-core kernel.
#include <cfloat>
#include <climits>
#include <mutex>
#include <type_traits>

#include "pa_common.cuh"
#include "pa_decode.h"
#include "pa_simt.cuh"
#include "pa_tc.cuh"

namespace pa {

namespace {

constexpr int kD = 128;
constexpr int kN = 16;              // MMA N of a 16-bit cache: query rows padded to 16
constexpr int kChunk = 128;         // tokens per chunk (MMA M)
constexpr int kChunkBlocks = kChunk / kBlock;
constexpr int kRegion = kChunk * 128;   // one 64-dim half of a 16-bit K or V tile, or one chunk of E4M3 codes (bytes)

// FP8 caches run both products on the E4M3 codes as loaded: Q is split into
// three E4M3 parts and P into four, stacked as 3G and 4G columns, so S has
// NSq = 3G columns rounded up to the MMA's N granule of 16 and O has NSo =
// 4G.  TMEM: four buffers (S twice, then O twice), each starting at a
// multiple of its power-of-two stride: 16 columns each for G = 4 (64 in
// all), 32 for G = 8 (128), 64 for G = 16 (256).
constexpr int kQParts = 3, kPParts = 4;
__host__ __device__ constexpr int round16(int x) { return (x + 15) / 16 * 16; }
__host__ __device__ constexpr int pow2_at_least(int x) { return x <= 16 ? 16 : x <= 32 ? 32 : x <= 64 ? 64 : 128; }
__host__ __device__ constexpr int tc_cols_s(int G, bool e4m3) { return e4m3 ? round16(kQParts * G) : kN; }
__host__ __device__ constexpr int tc_cols_o(int G, bool e4m3) { return e4m3 ? kPParts * G : kN; }
__host__ __device__ constexpr int tc_buf_stride(int nsq, int nso) { return pow2_at_least(nsq > nso ? nsq : nso); }
__host__ __device__ constexpr uint32_t tc_tmem_cols(int nsq, int nso) {
    return 4 * tc_buf_stride(nsq, nso) < 32 ? 32u : (uint32_t)(4 * tc_buf_stride(nsq, nso));
}
template <int NSq, int NSo>
__device__ __forceinline__ uint32_t s_col(int b) { return (uint32_t)(b * tc_buf_stride(NSq, NSo)); }
template <int NSq, int NSo>
__device__ __forceinline__ uint32_t o_col(int b) { return (uint32_t)((2 + b) * tc_buf_stride(NSq, NSo)); }
static_assert(tc_tmem_cols(16, 16) == 64 && tc_tmem_cols(32, 32) == 128 && tc_tmem_cols(48, 64) == 256,
              "TMEM columns per CTA");

// FP8 caches with 8 or 16 query rows per KV head take the "wide" shape: 8
// softmax warps (two per TMEM lane quadrant, each thread holding half the
// columns: the E4M3 weight split is the per-chunk work that sets the pace
// there) at 2 CTAs per SM, with three stages per operand.  With 4 rows the
// 3-CTA shape wins (measured: gqa8b over FP8 152 us against 188 us wide,
// long70b over FP8 175 us against 164 us wide): a batch of short
// sequences needs the third CTA per SM to cover each CTA's start.
__host__ __device__ constexpr bool tc_wide(int G, bool e4m3) { return G > 8 || (e4m3 && G >= 8); }

// K / V stages: a 16-bit chunk fills a 32 KiB tile area (two 64-dim
// regions), one stage per operand; E4M3 codes take 16 KiB a chunk, two
// stages per operand at 3 CTAs per SM, three with the wide FP8 shape, so
// the loads of the next chunks overlap the products and the softmax of the
// current one.
constexpr int kMaxStages = 3;
__host__ __device__ constexpr int tc_stages(int G, bool e4m3) { return !e4m3 ? 1 : tc_wide(G, e4m3) ? 3 : 2; }
// V stages: a second one for 16-bit caches with 16 columns, whose two CTAs
// per SM leave room for it; the V load of chunk c + 1 then overlaps the
// softmax and the PV product of chunk c instead of starting after them.
__host__ __device__ constexpr int tc_stages_v(int G, bool e4m3) { return !e4m3 && G > 8 ? 2 : tc_stages(G, e4m3); }
__host__ __device__ constexpr int tc_stage_bytes(bool e4m3) { return e4m3 ? kRegion : 2 * kRegion; }

// Shared-memory layout (bytes from the 1024-aligned base): K tile area,
// V tile area, Q tile (16-bit: two 64-dim regions of 16 rows; E4M3: NSq
// rows of 128 codes), P tile (16-bit: two 64-token regions of 16 rows;
// E4M3: NSo rows of 128 codes), the cross-warp reduction [2][4][16]
// floats, the mbarriers, TMEM base / fail flag / 4 lazy-max flags, and the
// per-row logit factors of the E4M3 path.
constexpr int kNumBars = 4 * kMaxStages + 6;
struct TcLayout {
    int k_off, v_off, q_off, p_off, red_off, bar_off, misc_off, qscale_off, bytes;
    __host__ __device__ constexpr TcLayout(int G, bool e4m3)
        : k_off(0), v_off(tc_stages(G, e4m3) * tc_stage_bytes(e4m3)),
          q_off((tc_stages(G, e4m3) + tc_stages_v(G, e4m3)) * tc_stage_bytes(e4m3)),
          p_off(q_off + (e4m3 ? tc_cols_s(G, true) * 128 : 2 * kN * 128)),
          red_off(p_off + (e4m3 ? tc_cols_o(G, true) * 128 : 2 * kN * 128)), bar_off(red_off + 2 * 4 * kN * 4),
          misc_off(bar_off + kNumBars * 8), qscale_off(misc_off + 32),
          bytes(qscale_off + kN * 4) {}
};

// Two fp32 values packed in one 64-bit register pair, and the sm_100
// packed arithmetic on them: each lane is the ordinary IEEE round-to-nearest
// single-precision operation, two per instruction.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 up2(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

__device__ __forceinline__ bool is_failed(const int *f) { return *reinterpret_cast<const volatile int *>(f) != 0; }

// Bounded wait that gives up at once when another thread already failed.
__device__ __forceinline__ bool wait_ok(uint64_t *bar, uint32_t parity, int *fail) {
    if (is_failed(fail)) return false;
    if (mbar_wait(bar, parity)) return true;
    atomicOr(fail, 1);
    return false;
}

// Maximum of v over the warp (NaN inputs ignored, like fmaxf), one
// instruction on sm_100a.
__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

// Named barrier 1 over the N softmax threads.
template <int N>
__device__ __forceinline__ void softmax_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// One producer warp streams one of the two tiles (K or V) chunk by chunk
// through kStages stages: wait until the MMA that read the stage's previous
// chunk has completed (`empty[stage]`), then load the chunk's 8 blocks
// (zeros past the partition) completing on `full[stage]`.  The table slice
// is held in registers, 32 entries per window, the next window prefetched
// one window ahead.  kCodes: the tile holds E4M3 codes, one 128-byte row per
// token (one box per block) instead of two 64-dim regions of 16-bit elements.
// The first two 32-entry windows of a producer's table slice, loaded before
// the context length is known (entries past the slice are read, when they
// lie inside the table row, and ignored).
struct TablePrefetch {
    bool valid;
    int32_t w0, w1;
};

template <bool kCodes, int kStages, int nheads>
__device__ __forceinline__ void produce_tile(const DecodeParams &p, const CUtensorMap *tmap, unsigned char *tile,
                                             uint64_t *full, uint64_t *empty, int *fail, int s, int kvh0, int b0,
                                             int nb, int nch, int oob_row, int lane, const TablePrefetch &pre) {
    constexpr int kStageBytes = tc_stage_bytes(kCodes);
    const int32_t *row = p.block_tables + (int64_t)s * p.max_blocks_per_seq + b0;
    auto slot_of = [&](int bi, int32_t entry, int kvh) -> int {
        return bi < nb ? (int)((checked_block(p, entry) * p.num_kv_heads + kvh) * kBlock) : oob_row;
    };
    auto window = [&](int w, int kvh) -> int {
        const int bi = w * 32 + lane;
        return slot_of(bi, bi < nb ? row[bi] : 0, kvh);
    };
    if (lane == 0) prefetch_tmap(tmap);
    int issued = 0;  // chunks issued, counted over all heads (stages and phases follow this count)
    bool ok = true;
    for (int h = 0; h < nheads && ok; ++h) {
        const int kvh = kvh0 + h;
        int cur = pre.valid ? slot_of(lane, pre.w0, kvh) : window(0, kvh);
        int next = nb > 32 ? (pre.valid ? slot_of(32 + lane, pre.w1, kvh) : window(1, kvh)) : oob_row;
        for (int c = 0; c < nch; ++c) {
            if (c > 0 && (c & 3) == 0) {
                cur = next;
                next = (c / 4 + 1) * 32 < nb ? window(c / 4 + 1, kvh) : oob_row;
            }
            const int y = __shfl_sync(0xffffffffu, cur, ((c & 3) << 3) + (lane & 7));
            const int cc = issued;
            const int st = cc % kStages;
            if (lane == 0) {
                ok = cc < kStages || wait_ok(&empty[st], (cc / kStages - 1) & 1, fail);
                if (ok) mbar_arrive_expect_tx(&full[st], kCodes ? kRegion : 2 * kRegion);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            unsigned char *dst = tile + st * kStageBytes;
            if (lane < kChunkBlocks) {
                tc::tma_load_2d(dst + lane * 2048, tmap, 0, y, &full[st]);
                if constexpr (!kCodes) tc::tma_load_2d(dst + kRegion + lane * 2048, tmap, 64, y, &full[st]);
            }
            issued = cc + 1;
        }
    }
    // After a failure the last chunks issued may still be landing (their
    // consumer gave up): give each a bounded chance before the CTA exits.
    // At most kStages chunks are outstanding: chunk c is issued only after
    // chunk c - kStages was consumed.
    if (lane == 0 && is_failed(fail))
        for (int c = issued - kStages > 0 ? issued - kStages : 0; c < issued; ++c)
            mbar_wait(&full[c % kStages], (c / kStages) & 1, 200000000ll);
}

// Softmax warps: one per TMEM lane quadrant, each thread holding the state
// of every column; with 16 columns two warps per quadrant, each owning 8 of
// the columns, so a thread's state stays that of 8 columns.  Then one more
// group of 4 warps: the K producer, the MMA issuer, the V producer and an
// idle warp.  The compiler caps registers as if a CTA's warps came in fours
// anyway (80 per thread for 3 CTAs of 7 or 8 warps per SM); with the fourth
// warp present it spills far less in the softmax loop (measured with
// -Xptxas -v: 44 -> 4 bytes for 8 columns).
__host__ __device__ constexpr int tc_soft_warps(int G, bool e4m3) { return tc_wide(G, e4m3) ? 8 : 4; }
__host__ __device__ constexpr int tc_threads(int G, bool e4m3) { return (tc_soft_warps(G, e4m3) + 4) * 32; }

// CTAs per SM: 3 (registers and shared memory both allow it) except with 16
// columns, whose 11 warps fit twice.
__host__ __device__ constexpr int tc_ctas_per_sm(int G, bool e4m3) { return tc_wide(G, e4m3) ? 2 : 3; }

// G: columns of S (query rows per KV head: the group, or group x query
// tokens with kMasked, padded to a power of two).
// kFp8: the caches hold E4M3 codes; k_scale sits in scale_log2 and v_scale
// multiplies the output.  Both products run E4M3 x E4M3 on the codes as
// loaded, two stages per tile: Q is split into three E4M3 parts with one
// power-of-two factor per query row (4 + 4 + 4 significant bits recover any
// finite 16-bit q to within 2^-15 of the row's largest |q|), P into four
// parts (|w - sum| <= 2^-12 w + 2^-22); the f32 products of the parts are
// recombined when S and O are read from TMEM.
// kHpc: KV heads one CTA streams (2 only for plain 16-bit decode with G * 2
// <= 16 query rows; with 1 the head bookkeeping compiles away).
template <typename T, int G, bool kMasked, bool kFp8, int kHpc = 1>
__global__ void __launch_bounds__(tc_threads(G, kFp8), tc_ctas_per_sm(G, kFp8))
    decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const int oob_row) {
    static_assert(!kFp8 || kMasked, "FP8 launches take the masked variant (it applies v_scale)");
    static_assert(kHpc == 1 || (!kMasked && G * kHpc <= kN), "several heads per CTA: plain decode, 16 rows");
    using E = Elem<T>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr int kSW = tc_soft_warps(G, kFp8);  // softmax warps
    constexpr int kST = kSW * 32;                // softmax threads
    constexpr int kGT = tc_soft_warps(G, kFp8) == 8 ? G / 2 : G;  // columns per softmax thread
    constexpr int kWarpK = kSW, kWarpMma = kSW + 1, kWarpV = kSW + 2;
    constexpr bool kE4m3 = kFp8;                 // both products on the E4M3 codes
    constexpr int kNSq = tc_cols_s(G, kE4m3);    // columns of S
    constexpr int kNSo = tc_cols_o(G, kE4m3);    // columns of O
    constexpr uint32_t kTmemCols = tc_tmem_cols(kNSq, kNSo);
    constexpr int kStages = tc_stages(G, kE4m3);      // K stages
    constexpr int kStagesV = tc_stages_v(G, kE4m3);   // V stages
    constexpr int kStageBytes = tc_stage_bytes(kE4m3);
    constexpr TcLayout Lay(G, kE4m3);
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *k_t = smem + Lay.k_off;
    unsigned char *v_t = smem + Lay.v_off;
    unsigned char *q_t = smem + Lay.q_off;
    unsigned char *p_t = smem + Lay.p_off;
    float *red = reinterpret_cast<float *>(smem + Lay.red_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay.bar_off);
    uint64_t *k_full = bars, *k_empty = bars + kMaxStages;  // [kStages]
    uint64_t *v_full = bars + 2 * kMaxStages, *v_empty = bars + 3 * kMaxStages;
    uint64_t *s_full = bars + 4 * kMaxStages, *o_full = s_full + 2, *p_full = s_full + 4, *q_full = s_full + 5;
    float *qscale = reinterpret_cast<float *>(smem + Lay.qscale_off);  // kE4m3: logit factor per query row
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay.misc_off);
    int *fail = reinterpret_cast<int *>(smem + Lay.misc_off + 4);
    int *lazy_flag = reinterpret_cast<int *>(smem + Lay.misc_off + 8);  // [4], by chunk & 3

    // this CTA streams KV heads kvh .. kvh + hpc - 1 (plain decode only: the
    // query rows of hpc heads, G each, fill the Q tile's 16 rows) and, for
    // each, partitions part0 .. part0 + ppc - 1 (those that exist), back to
    // back: one set-up, one pipeline, one partial per (head, partition)
    constexpr int hpc = kHpc;
    // Grid: x = partition group, y = KV head group, z = schedule position (a
    // sequence's CTAs launch together), or with p.part_major x = KV head
    // group, y = schedule position, z = partition group (every sequence's
    // first partition launches before any later one)
    const bool pm = p.part_major != 0;
    const int g_part = pm ? (int)blockIdx.z : (int)blockIdx.x;
    const int g_head = pm ? (int)blockIdx.x : (int)blockIdx.y;
    const int g_seq = pm ? (int)blockIdx.y : (int)blockIdx.z;
    const int kvh = g_head * hpc;
    const int ppc = p.parts_per_cta;
    const int part0 = g_part * ppc;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.num_heads, head0 = kvh * G;  // head0: unmasked launches (group == G, q_len == 1)
    T *out = reinterpret_cast<T *>(p.out);
    pdl_launch_dependents();
    // Until pdl_wait() below the CTA reads only inputs that no kernel of this
    // library writes (seq_order, block table, context length, q), so this
    // part overlaps the tail of the kernel before it on the stream; the
    // caches, the output and the workspace are touched after the wait.
    const int s = scheduled_seq(p, g_seq, part0 == 0 && g_head == 0 && tid == 0);
    if (s < 0) return;
    // Without a window a CTA's slice of the table starts at part0 *
    // part_blocks whatever the context length: the producers issue its first
    // two windows now, so their latency overlaps the length load and the
    // set-up below.
    TablePrefetch pre{false, 0, 0};
    if ((warp == kWarpK || warp == kWarpV) && p.window <= 0) {
        const int32_t *row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
        const int bi = part0 * p.part_blocks + lane;
        pre.valid = true;
        if (bi < p.max_blocks_per_seq) pre.w0 = row[bi];
        if (bi + 32 < p.max_blocks_per_seq) pre.w1 = row[bi + 32];
    }
    // flat q / out row of row r: plain decode keeps the group's rows contiguous
    auto row_of = [&](int r) -> int64_t {
        if constexpr (kMasked) return query_row(p, s, kvh, r);
        return (int64_t)s * H + head0 + r;
    };
    const int rows = kMasked ? p.group * p.q_len : G * hpc;  // real Q rows of the CTA

    const SeqSplit sp = seq_split(p, s, part0 == 0 && g_head == 0 && tid == 0);
    const int L = sp.L, nblk = sp.nblk, nparts = sp.nparts;
    if (part0 >= nparts) return;
    const int nmine = min(ppc, nparts - part0);  // partitions of this CTA
    const bool direct = nparts == 1;
    // The softmax warps load their query rows now, before the set-up: E4M3,
    // a warp per row (rows warp, warp + kSW, ..), 4 dims per lane; 16-bit,
    // 16-byte pieces (piece i: row i / 16, dims 8 (i % 16) ..)
    constexpr int kQRowsW = kE4m3 ? (G + kSW - 1) / kSW : 1;
    constexpr int kQPieces = kE4m3 ? 1 : (kN * (kD / 8) + kST - 1) / kST;
    uint2 q8[kQRowsW];
    uint4 q16[kQPieces];
    if (warp < kSW) {
        const T *q = reinterpret_cast<const T *>(p.q);
        if constexpr (kE4m3) {
#pragma unroll
            for (int k = 0; k < kQRowsW; ++k) {
                const int r = warp + k * kSW;
                q8[k] = r < G && r < rows ? *reinterpret_cast<const uint2 *>(q + row_of(r) * kD + 4 * lane)
                                          : make_uint2(0, 0);
            }
        } else {
#pragma unroll
            for (int k = 0; k < kQPieces; ++k) {
                const int i = tid + k * kST, r = i / (kD / 8);
                q16[k] = i < kN * (kD / 8) && r < rows
                             ? *reinterpret_cast<const uint4 *>(q + row_of(r) * kD + (i % (kD / 8)) * 8)
                             : make_uint4(0, 0, 0, 0);
            }
        }
    }
    pdl_wait();
    if (L == 0) {
        for (int i = tid; i < rows * kD; i += blockDim.x) out[row_of(i / kD) * kD + i % kD] = E::from_float(0.f);
        return;
    }
    // The swizzled tiles need a 1024-byte aligned base; never touch them otherwise.
    if (smem_addr(smem) & 1023u) {
        if (tid == 0) flag_error(PA_DEVERR_LAYOUT);
        return;
    }
    const int b0 = sp.bfirst + part0 * p.part_blocks;
    const int nb = min(nmine * p.part_blocks, nblk - b0);  // blocks of this CTA's partitions
    const int nch = (nb + kChunkBlocks - 1) / kChunkBlocks; // chunks of 128 tokens
    // One partial per CTA: the partitions a CTA streams (ppc > 1 only when
    // they start on a chunk) are combined into the slot of its first one,
    // and the others are marked empty (lse = -inf, weight 0 in the merge),
    // so the pipeline runs through partition boundaries instead of draining
    // at each.  cpp: chunks per written partial, all of a head's chunks.
    const int cpp = nch;
    const int tok0 = b0 * kBlock;
    const int tok_end = min(L, (b0 + nb) * kBlock);         // tokens of this CTA: [tok0, tok_end)
    const int nct = hpc * nch;                              // chunks of all the CTA's heads

    // ---- set-up -----------------------------------------------------------------
    if (warp == kWarpMma) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        *fail = 0;
        for (int i = 0; i < 4; ++i) lazy_flag[i] = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < kStagesV; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(&o_full[0], 1);
        mbar_init(&o_full[1], 1);
        mbar_init(p_full, kST);
        mbar_init(q_full, kST);
        fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpK) {
        produce_tile<kE4m3, kStages, kHpc>(p, &tmap_k, k_t, k_full, k_empty, fail, s, kvh, b0, nb, nch, oob_row,
                                           lane, pre);
    } else if (warp == kWarpV) {
        produce_tile<kE4m3, kStagesV, kHpc>(p, &tmap_v, v_t, v_full, v_empty, fail, s, kvh, b0, nb, nch, oob_row,
                                           lane, pre);
    } else if (warp == kWarpMma) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc_qk =
                kE4m3 ? tc::instr_desc_e4m3(false, kChunk, kNSq) : tc::instr_desc_f16(kBf16, false, kChunk, kN);
            constexpr uint32_t idesc_pv =
                kE4m3 ? tc::instr_desc_e4m3(true, kD, kNSo) : tc::instr_desc_f16(kBf16, true, kD, kN);
            const uint32_t kb = smem_addr(k_t), vb = smem_addr(v_t), qb = smem_addr(q_t), pb = smem_addr(p_t);
            // PV(c): O^T = V^T . P^T into O buffer c & 1
            auto issue_pv = [&](int c) {
                const int st = c % kStagesV;
                tc::fence_after_sync();
                const uint32_t vs = vb + st * kStageBytes;
                if constexpr (kE4m3) {
                    // V codes MN-major (a token's 128 dims are one 128-byte atom row),
                    // 32 tokens per MMA; P parts K-major, one 128-byte row per column
#pragma unroll
                    for (int kk = 0; kk < kChunk / 32; ++kk) {
                        const uint64_t a = tc::smem_desc(vs + kk * 4096, kRegion, 1024);
                        const uint64_t b = tc::smem_desc(pb + kk * 32, 16, 1024);
                        tc::mma_e4m3(tmem + o_col<kNSq, kNSo>(c & 1), a, b, idesc_pv, kk > 0);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < kChunk / 16; ++kk) {
                        const uint64_t a = tc::smem_desc(vs + kk * 2048, kRegion, 1024);
                        const uint64_t b = tc::smem_desc(pb + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024);
                        tc::mma_f16(tmem + o_col<kNSq, kNSo>(c & 1), a, b, idesc_pv, kk > 0);
                    }
                }
                tc::commit(&o_full[c & 1]);
                tc::commit(&v_empty[st]);
            };
            // S(c) = K . Q^T into S buffer c & 1
            auto issue_s = [&](int c) {
                const int st = c % kStages;
                tc::fence_after_sync();
                const uint32_t ks = kb + st * kStageBytes;
                if constexpr (kE4m3) {
                    // K codes: one 128-byte row per token; Q parts: one 128-byte row per column
#pragma unroll
                    for (int kk = 0; kk < kD / 32; ++kk) {
                        const uint64_t a = tc::smem_desc(ks + kk * 32, 16, 1024);
                        const uint64_t b = tc::smem_desc(qb + kk * 32, 16, 1024);
                        tc::mma_e4m3(tmem + s_col<kNSq, kNSo>(c & 1), a, b, idesc_qk, kk > 0);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint64_t a = tc::smem_desc(ks + (kk >> 2) * kRegion + (kk & 3) * 32, 16, 1024);
                        const uint64_t b = tc::smem_desc(qb + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024);
                        tc::mma_f16(tmem + s_col<kNSq, kNSo>(c & 1), a, b, idesc_qk, kk > 0);
                    }
                }
                tc::commit(&s_full[c & 1]);
                tc::commit(&k_empty[st]);
            };
            // The two products are issued in whichever order their inputs
            // arrive, polled without blocking: S(n) once K(n) has landed and
            // PV(n - 2) is issued (S(n) reuses the TMEM buffer of S(n - 2),
            // which the softmax warps read before handing over P(n - 2));
            // PV(n) once P(n) and V(n) are there.  A late K never holds back
            // a ready PV, nor a late P a ready S.  Bounded like every wait.
            bool ok = wait_ok(q_full, 0, fail);
            int ns = 0, npv = 0;
            long long t_last = clock64();
            while (ok && npv < nct) {
                bool progress = false;
                if (ns < nct && ns <= npv + 1 && mbar_test(&k_full[ns % kStages], (ns / kStages) & 1)) {
                    issue_s(ns);
                    ++ns;
                    progress = true;
                }
                if (npv < ns && mbar_test(p_full, npv & 1) &&
                    mbar_test(&v_full[npv % kStagesV], (npv / kStagesV) & 1)) {
                    issue_pv(npv);
                    ++npv;
                    progress = true;
                }
                if (progress) {
                    t_last = clock64();
                } else if (is_failed(fail)) {
                    ok = false;
                } else if (clock64() - t_last > kWaitLimitCycles) {
                    flag_error(PA_DEVERR_TIMEOUT);
                    atomicOr(fail, 1);
                    ok = false;
                } else {
                    __nanosleep(32);
                }
            }
        }
        __syncwarp();
    } else if (warp < kSW) {
        // ------------------------------ softmax warps ------------------------------
        {
            // Q tile (rows loaded before the set-up), written while the
            // producers already stream K and V.
            if constexpr (kE4m3) {
                // Q as E4M3 parts, one warp per query row r, lane l holding
                // dims 4l .. 4l + 3: y = q * 2^e with max |y| in [128, 256),
                // hi = E4M3(y), mid = E4M3(16 (y - hi)), lo = E4M3(16 (16 (y - hi) - mid)),
                // so q = 2^-e (hi + mid / 16 + lo / 256) + err, |err| <= 2^-15 max |q|.
                // Rows hi: r, mid: G + r, lo: 2G + r of the 128-byte-swizzled
                // tile; padding rows zero.  qscale[r] = scale_log2 * 2^-e.
#pragma unroll
                for (int kr = 0; kr < kQRowsW; ++kr) {
                    const int r = warp + kr * kSW;
                    if (r >= G) break;  // warp-uniform
                    float y[4];
                    {
                        const float2 a = E::to_float2(q8[kr].x), b = E::to_float2(q8[kr].y);  // 0 past rows
                        y[0] = a.x;
                        y[1] = a.y;
                        y[2] = b.x;
                        y[3] = b.y;
                    }
                    float mx = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    const bool finite = mx <= FLT_MAX;  // false for inf and NaN
                    int e = 0;
                    if (mx > 0.f && finite) {
                        int k;
                        (void)frexpf(mx, &k);  // mx in [2^(k-1), 2^k)
                        e = 8 - k;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) y[i] = ldexpf(y[i], e);
#pragma unroll
                    for (int part = 0; part < kQParts; ++part) {
                        const uint16_t c01 = float2_to_e4m3x2(y[0], y[1]), c23 = float2_to_e4m3x2(y[2], y[3]);
                        *reinterpret_cast<uint32_t *>(q_t + tc::sw128_offset8(part * G + r, 4 * lane)) =
                            (uint32_t)c01 | ((uint32_t)c23 << 16);
                        const float2 d01 = e4m3x2_to_float2(c01), d23 = e4m3x2_to_float2(c23);
                        y[0] = (y[0] - d01.x) * 16.f;  // exact: the rounding error of y
                        y[1] = (y[1] - d01.y) * 16.f;
                        y[2] = (y[2] - d23.x) * 16.f;
                        y[3] = (y[3] - d23.y) * 16.f;
                    }
                    if (lane == 0) qscale[r] = finite ? ldexpf(p.scale_log2, -e) : NAN;
                }
                for (int r = kQParts * G + warp; r < kNSq; r += kSW)  // padding columns
                    *reinterpret_cast<uint32_t *>(q_t + tc::sw128_offset8(r, 4 * lane)) = 0u;
            } else {
                // rows = the group's query heads (zero rows up to 16), K-major
                // 128-byte swizzle, two 64-dim regions
#pragma unroll
                for (int k = 0; k < kQPieces; ++k) {
                    const int i = tid + k * kST;
                    if (i >= kN * (kD / 8)) break;
                    const int r = i / (kD / 8), c16 = i % (kD / 8);  // row, 16-byte chunk
                    *reinterpret_cast<uint4 *>(q_t + (c16 >> 3) * (kN * 128) + tc::sw128_offset(r, (c16 & 7) * 8)) =
                        q16[k];
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(q_full);
            if constexpr (kE4m3) softmax_sync<kST>();  // qscale written by every softmax warp
        }
        const int t = tid & 127;                                      // token of S, dim of O
        const int c0 = kSW == 8 ? (warp >> 2) * kGT : 0;              // this thread's first column
        const uint32_t lane_base = (uint32_t)((kSW == 8 ? warp & 3 : warp) * 32) << 16;  // TMEM lane quadrant
        // masked launches: column h is query token h >> lg, whose position is
        // hi0 + (h >> lg); it attends (position - window, position] (all
        // positions up to its own without a window); padding columns none
        const int hi0 = L - p.q_len;
        const int lg = 31 - __clz(p.group);
        const int win = p.window > 0 ? p.window : INT_MAX;
        // E4M3 products: column c0 + j of the result = sum over parts k of
        // TMEM column k G + c0 + j divided by 16^k (Horner from the last part)
        auto ld_parts = [&](auto np, uint32_t taddr, float *v) {
            constexpr int NP = decltype(np)::value;
            const uint64_t sixteenth = pk2(0.0625f, 0.0625f);
            if constexpr (G == 4) {
                float t16[16];
                tc::tmem_ld<16>(taddr, t16);
#pragma unroll
                for (int j = 0; j < kGT; j += 2) {
                    uint64_t a = pk2(t16[(NP - 1) * 4 + c0 + j], t16[(NP - 1) * 4 + c0 + j + 1]);
#pragma unroll
                    for (int k = NP - 2; k >= 0; --k)
                        a = fma2(a, sixteenth, pk2(t16[k * 4 + c0 + j], t16[k * 4 + c0 + j + 1]));
                    const float2 r = up2(a);
                    v[j] = r.x;
                    v[j + 1] = r.y;
                }
            } else {
                float b[kGT];
                uint64_t a[kGT / 2];
#pragma unroll
                for (int k = NP - 1; k >= 0; --k) {
                    tc::tmem_ld<kGT>(taddr + G * k + c0, b);
#pragma unroll
                    for (int j = 0; j < kGT; j += 2)
                        a[j / 2] = k == NP - 1 ? pk2(b[j], b[j + 1]) : fma2(a[j / 2], sixteenth, pk2(b[j], b[j + 1]));
                }
#pragma unroll
                for (int j = 0; j < kGT; j += 2) {
                    const float2 r = up2(a[j / 2]);
                    v[j] = r.x;
                    v[j + 1] = r.y;
                }
            }
        };
        // per-thread state of columns c0 + j, j < kGT
        float m[kGT], l[kGT], acc[kGT], alpha_prev[kGT];
#pragma unroll
        for (int j = 0; j < kGT; ++j) {
            m[j] = -INFINITY;
            l[j] = 0.f;
            acc[j] = 0.f;
            alpha_prev[j] = 1.f;
        }
        auto wait_o = [&](int c) { return wait_ok(&o_full[c & 1], (c >> 1) & 1, fail); };
        // O of chunk c (CTA-wide chunk count) of the head whose query rows
        // start at Q-tile row hgc
        auto load_o = [&](int c, int hgc) {
            tc::fence_after_sync();
            float o[8];
            if constexpr (kE4m3)
                ld_parts(std::integral_constant<int, kPParts>{}, tmem + lane_base + o_col<kNSq, kNSo>(c & 1), o);
            else
                tc::tmem_ld<kGT>(tmem + lane_base + o_col<kNSq, kNSo>(c & 1) + hgc + c0, o);
#pragma unroll
            for (int j = 0; j < kGT; ++j) acc[j] = fmaf(acc[j], alpha_prev[j], o[j]);
        };
        auto epilogue = [&](int c, int hgc) {
            if (wait_o(c)) load_o(c, hgc);
        };
        const bool has_tail = (b0 + nb == nblk) && (L % kBlock) != 0;  // partial last block here
        // the partial (pi = 0, in partition part0's slot) of head kvh + hh: per-column
        // sums over the 4 lane quadrants, then o = acc / l (and lse) to the
        // output or the workspace; the last sync frees `red` for the next
        // chunk's maxima (fewer syncs made the compiler spill in the loop)
        auto finalize = [&](int hh, int pi) {
            float *rl = red;
            softmax_sync<kST>();
#pragma unroll
            for (int j = 0; j < kGT; ++j) {
                float v = l[j];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) rl[(kSW == 8 ? warp & 3 : warp) * kN + c0 + j] = v;
            }
            softmax_sync<kST>();
            const int part = part0 + pi;
            if (!is_failed(fail)) {
#pragma unroll
                for (int j = 0; j < kGT; ++j) {
                    const int h = c0 + j;
                    const float lt = rl[h] + rl[kN + h] + rl[2 * kN + h] + rl[3 * kN + h];
                    if constexpr (kMasked) {
                        if (h >= rows) break;
                        // lt = 0 only for a column with no position in this partition
                        const float o = lt > 0.f ? acc[j] / lt * p.v_scale : 0.f;
                        const int64_t qr = row_of(h);
                        if (direct) {
                            out[qr * kD + t] = E::from_float(o);
                        } else {
                            const int64_t r = qr * p.max_parts + part;
                            p.ws_o[r * kD + t] = o;
                            if (t == 0) {
                                p.ws_lse[r] = lt > 0.f ? m[j] + log2f(lt) : -INFINITY;
                                for (int k = 1; k < nmine; ++k) p.ws_lse[r + k] = -INFINITY;
                            }
                        }
                    } else {  // plain decode: every column has tokens, V unscaled
                        const float o = acc[j] / lt;
                        const int64_t qh = (int64_t)s * H + head0 + hh * G + h;  // query head of column h
                        if (direct) {
                            out[qh * kD + t] = E::from_float(o);
                        } else {
                            const int64_t r = qh * p.max_parts + part;
                            p.ws_o[r * kD + t] = o;
                            if (t == 0) {
                                p.ws_lse[r] = m[j] + log2f(lt);
                                for (int k = 1; k < nmine; ++k) p.ws_lse[r + k] = -INFINITY;
                            }
                        }
                    }
                }
            }
            softmax_sync<kST>();
        };
        int hh = 0, cbase = 0;  // the head of chunk cc, and the CTA-wide index of its first chunk
        for (int cc = 0; cc < nct; ++cc) {
            float x[kGT];
            if constexpr (kHpc > 1) {
                if (cc - cbase == nch) {
                    cbase += nch;
                    ++hh;
                }
            }
            const int c = cc - cbase;  // this head's chunk
            const int hg = hh * G;     // its first query row in the Q tile
            const int tok = tok0 + c * kChunk + t;
            const int cl = c % cpp;  // chunk index within its partition
            if (cl == 0 && cc > 0) {
                // chunk cc - 1 closed a partition (or a head): finish and write it, start afresh
                const int hp = c == 0 ? hh - 1 : hh;
                epilogue(cc - 1, hp * G);
                finalize(hp, c == 0 ? (nch - 1) / cpp : c / cpp - 1);
#pragma unroll
                for (int j = 0; j < kGT; ++j) {
                    m[j] = -INFINITY;
                    l[j] = 0.f;
                    acc[j] = 0.f;
                    alpha_prev[j] = 1.f;
                }
            }
            const bool valid = tok < tok_end;
            bool ok = wait_ok(&s_full[cc & 1], (cc >> 1) & 1, fail);
            bool exceed = false;
            if (ok) {
                tc::fence_after_sync();
                float sv[8];
                const uint32_t sb = tmem + lane_base + s_col<kNSq, kNSo>(cc & 1);
                float scl[kGT];
                if constexpr (kE4m3) {
                    ld_parts(std::integral_constant<int, kQParts>{}, sb, sv);
#pragma unroll
                    for (int j = 0; j < kGT; ++j) scl[j] = qscale[c0 + j];
                } else {
                    tc::tmem_ld<kGT>(sb + hg + c0, sv);
#pragma unroll
                    for (int j = 0; j < kGT; ++j) scl[j] = p.scale_log2;
                }
#pragma unroll
                for (int j = 0; j < kGT; ++j) {
                    bool live = valid;
                    if constexpr (kMasked) {
                        const int h = c0 + j;
                        const int pos = hi0 + (h >> lg);
                        live = live && h < rows && tok <= pos && pos - tok < win;
                    }
                    x[j] = live ? sv[j] * scl[j] : -INFINITY;
                    exceed |= x[j] > m[j] + kLazyMax;
                }
            } else {
#pragma unroll
                for (int j = 0; j < kGT; ++j) x[j] = -INFINITY;
            }
            // Lazy running max: a CTA-wide flag says whether any logit of the
            // chunk beats its head's running max by more than 2^8; only then
            // are the per-head chunk maxima reduced and the state rescaled.
            if (__any_sync(0xffffffffu, exceed) && lane == 0) lazy_flag[cc & 3] = 1;
            softmax_sync<kST>();
            const bool update = lazy_flag[cc & 3] != 0;
            if (tid == 0) lazy_flag[(cc + 2) & 3] = 0;  // slot of chunk cc + 2: its readers are done
            float alpha[kGT];
#pragma unroll
            for (int j = 0; j < kGT; ++j) alpha[j] = 1.f;
            if (update) {  // uniform across the softmax threads
                float *rc = red + (cc & 1) * 4 * kN;  // [quadrant][column]
#pragma unroll
                for (int j = 0; j < kGT; ++j) {
                    const float v = warp_max(x[j]);
                    if (lane == 0) rc[(kSW == 8 ? warp & 3 : warp) * kN + c0 + j] = v;
                }
                softmax_sync<kST>();
#pragma unroll
                for (int j = 0; j < kGT; ++j) {
                    const int h = c0 + j;
                    const float cm = fmaxf(fmaxf(rc[h], rc[kN + h]), fmaxf(rc[2 * kN + h], rc[3 * kN + h]));
                    if (cm > m[j] + kLazyMax) {
                        alpha[j] = ex2(m[j] - cm);  // 0 on the first chunk (m = -inf)
                        l[j] *= alpha[j];
                        m[j] = cm;
                    }
                }
            }
            T pv[kGT];
            uint16_t pc[kPParts][kGT / 2];  // E4M3: the weights' parts, two columns per code pair
            if constexpr (kE4m3) {
                // w = sum over k of part_k / 16^k, part_0 = E4M3(w), part_k = E4M3(16 r_k) with
                // r_k the remainder after part k - 1; w <= 2^8 (the lazy max), so no part
                // saturates, and |w - sum| <= 2^-12 w + 2^-22
#pragma unroll
                for (int j = 0; j < kGT; j += 2) {
                    // a masked column may still have m = -inf: weight 0, not 2^(-inf + inf)
                    const float a = x[j] == -INFINITY ? 0.f : ex2(x[j] - m[j]);
                    const float b = x[j + 1] == -INFINITY ? 0.f : ex2(x[j + 1] - m[j + 1]);
                    // the pair (a, b) in one register pair: remainder r, sums w
                    uint64_t r = pk2(a, b), w = pk2(0.f, 0.f);
                    float f = 1.f;
#pragma unroll
                    for (int k = 0; k < kPParts; ++k) {
                        const float2 rf = up2(r);
                        const uint16_t code = float2_to_e4m3x2(rf.x, rf.y);
                        const float2 d = e4m3x2_to_float2(code);
                        const uint64_t dd = pk2(d.x, d.y);
                        pc[k][j / 2] = code;
                        w = fma2(dd, pk2(f, f), w);
                        r = mul2(sub2(r, dd), pk2(16.f, 16.f));  // exact: the part's rounding error, scaled
                        f *= 0.0625f;
                    }
                    const float2 wf = up2(w);
                    l[j] += wf.x;  // the weight the MMA sees (to f32 rounding)
                    l[j + 1] += wf.y;
                }
            } else {
#pragma unroll
                for (int j = 0; j < kGT; ++j) {
                    // a masked column may still have m = -inf: weight 0, not 2^(-inf + inf)
                    pv[j] = (kMasked && x[j] == -INFINITY) ? E::from_float(0.f) : E::from_float(ex2(x[j] - m[j]));
                    l[j] += E::to_float(pv[j]);  // the rounded weight the MMA sees
                }
            }
            const bool o_prev = cl > 0 && wait_o(cc - 1);
            if (c == nch - 1 && has_tail && ok && c0 == 0) {
                // Rows of the partial last block past the context come from the
                // pool and may hold anything (NaN): zero them in the V tile
                // once it has landed, so 0 * V stays 0 in the PV product.
                const int st = cc % kStagesV;
                unsigned char *vt = v_t + st * kStageBytes;
                if (wait_ok(&v_full[st], (cc / kStagesV) & 1, fail) && tok >= L && tok < (b0 + nb) * kBlock) {
#pragma unroll
                    for (int j = 0; j < (kE4m3 ? 1 : 2); ++j)  // E4M3: a token's codes are one 128-byte row
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            *reinterpret_cast<uint4 *>(vt + j * kRegion + t * 128 + k * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            // P tile: K-major, rows = columns of O, 128-byte rows of tokens
            if constexpr (kE4m3) {
                // E4M3 part tile: part k of column c0 + j in row k G + c0 + j
#pragma unroll
                for (int k = 0; k < kPParts; ++k)
#pragma unroll
                    for (int j = 0; j < kGT; ++j)
                        p_t[tc::sw128_offset8(k * G + c0 + j, t)] = (unsigned char)(pc[k][j / 2] >> (8 * (j & 1)));
            } else {
                // two 64-token regions; this thread writes rows c0 .. c0 +
                // (16 / (kSW / 4)) - 1: its columns of the chunk's head (rows
                // hg .. hg + kGT - 1), zeros in the other rows
                unsigned char *pr = p_t + (t >> 6) * (kN * 128);
                constexpr int kRowsW = kN / (kSW / 4);
#pragma unroll
                for (int j = 0; j < kRowsW; ++j) {
                    T v = E::from_float(0.f);
#pragma unroll
                    for (int jj = 0; jj < kGT; ++jj)
                        if (j == hg + jj) v = pv[jj];
                    *reinterpret_cast<T *>(pr + tc::sw128_offset(c0 + j, t & 63)) = v;
                }
            }
            fence_proxy_async_smem();
            tc::fence_before_sync();
            mbar_arrive(p_full);
            if (o_prev) load_o(cc - 1, hg);
#pragma unroll
            for (int j = 0; j < kGT; ++j) alpha_prev[j] = alpha[j];
        }
        epilogue(nct - 1, hh * G);
        finalize(hh, (nch - 1) / cpp);
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kWarpMma) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// A cache [NB, Hk, 16, 128] seen as rows of 128 elements; boxes of 16 rows
// x 64 elements with the 128-byte swizzle; out-of-range rows read as zero.
// An FP8 cache [NB, Hk, 16, 128] seen as rows of 128 one-byte codes; boxes
// of 16 rows x 128 bytes with the 128-byte swizzle the MMA reads.
bool encode_code_map(CUtensorMap *map, const void *base, int64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kD};
    const cuuint32_t box[2] = {(cuuint32_t)kD, (cuuint32_t)kBlock};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_cache_map(CUtensorMap *map, const void *base, int64_t rows, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kBlock};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int G, bool kMasked, bool kFp8 = false, int kHpc = 1>
cudaError_t launch_tc_t(const DecodeParams &p, cudaStream_t stream) {
    const int64_t rows = p.num_blocks * p.num_kv_heads * kBlock;
    CUtensorMap tk, tv;
    const bool ok = kFp8 ? encode_code_map(&tk, p.k_cache, rows) && encode_code_map(&tv, p.v_cache, rows)
                         : encode_cache_map(&tk, p.k_cache, rows, std::is_same<T, __nv_bfloat16>::value) &&
                               encode_cache_map(&tv, p.v_cache, rows, std::is_same<T, __nv_bfloat16>::value);
    if (!ok) return cudaErrorInvalidValue;
    auto kern = decode_tc_kernel<T, G, kMasked, kFp8, kHpc>;
    static FuncAttrCache attrs;
    constexpr int kSmem = TcLayout(G, kFp8).bytes;
    static_assert(kSmem * tc_ctas_per_sm(G, kFp8) + 1024 * tc_ctas_per_sm(G, kFp8) <= 228 * 1024,
                  "the CTAs per SM must fit in shared memory");
    cudaError_t e = ensure_smem(kern, kSmem, attrs, /*max_carveout=*/true);
    if (e != cudaSuccess) return e;
    if (p.heads_per_cta != kHpc || p.num_kv_heads % kHpc != 0) return cudaErrorInvalidValue;
    const unsigned parts = (p.max_parts + p.parts_per_cta - 1) / p.parts_per_cta, heads = p.num_kv_heads / kHpc;
    if (p.part_major && parts > 65535) return cudaErrorInvalidValue;
    const dim3 grid = p.part_major ? dim3(heads, p.num_seqs, parts) : dim3(parts, heads, p.num_seqs);
    e = launch_pdl(kern, grid, dim3(tc_threads(G, kFp8)), kSmem, stream, p, tk, tv, (int)rows);
    if (e != cudaSuccess || p.max_parts == 1) return e;
    return launch_merge_partitions(p, std::is_same<T, __nv_bfloat16>::value ? PA_BF16 : PA_F16, kD, stream);
}

template <typename T, bool kMasked>
cudaError_t launch_tc_m(const DecodeParams &p, int rows, cudaStream_t stream) {
    if constexpr (!kMasked) {
        if (p.heads_per_cta == 2) {  // two KV heads per CTA (plain decode, groups of 4 or 8)
            switch (rows) {
                case 4: return launch_tc_t<T, 4, false, false, 2>(p, stream);
                case 8: return launch_tc_t<T, 8, false, false, 2>(p, stream);
                default: return cudaErrorInvalidValue;
            }
        }
    }
    switch (rows) {
        case 4: return launch_tc_t<T, 4, kMasked>(p, stream);
        case 8: return launch_tc_t<T, 8, kMasked>(p, stream);
        case 16: return launch_tc_t<T, 16, kMasked>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

// The plain variant neither masks nor scales V: anything else takes the
// masked one (with q_len = 1, no window its masks keep every token).
template <typename T>
cudaError_t launch_tc_fp8(const DecodeParams &p, int rows, cudaStream_t stream) {
    switch (rows) {
        case 4: return launch_tc_t<T, 4, true, true>(p, stream);
        case 8: return launch_tc_t<T, 8, true, true>(p, stream);
        case 16: return launch_tc_t<T, 16, true, true>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_tc_d(const DecodeParams &p, int rows, bool fp8, cudaStream_t stream) {
    if (fp8) return launch_tc_fp8<T>(p, rows, stream);
    return decode_masked(p) || p.v_scale != 1.f ? launch_tc_m<T, true>(p, rows, stream)
                                                : launch_tc_m<T, false>(p, rows, stream);
}

}  // namespace

bool decode_tc_supported(int head_dim, int rows, int64_t num_blocks, int num_kv_heads) {
    return head_dim == kD && (rows == 4 || rows == 8 || rows == 16) &&
           num_blocks * num_kv_heads * kBlock < ((int64_t)1 << 31) - kBlock;
}

cudaError_t launch_decode_tc(const DecodeParams &p, int dtype, int rows, bool fp8_cache, cudaStream_t stream) {
    return dtype == PA_F16 ? launch_tc_d<__half>(p, rows, fp8_cache, stream)
                           : launch_tc_d<__nv_bfloat16>(p, rows, fp8_cache, stream);
}

}  // namespace pa
