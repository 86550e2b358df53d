// Block-sparse exact softmax attention over selected key clusters (AdaCluster,
// Algorithm 3's sparse attention; its dense branch for dense heads), bf16 inputs, two query tiles
// per CTA, 128-key chunks.
//
// A work item is up to 256 query rows of one query cluster (two 128-row
// tiles) that share one key stream (KeyStream): the rows of the cluster's key
// runs packed into chunks of 128 keys, loaded by TMA into K and V rings.
// TMEM holds, per tile t, one S buffer of 128 columns and the O accumulator:
//   S_0 | S_1 | O_0 | O_1   (128 + 128 + 2 D columns).
// Softmax warpgroup t turns S_t(j) into P_t(j) (bf16, written back over the
// first 64 columns of S_t, two keys per column).  The single MMA thread
// issues, per chunk j and tile t in turn,
//   O_t += P_t(j) V_j            (A operand read from TMEM) once P_t(j) is written,
//   S_t(j+1) = Q_t K_{j+1}^T     into S_t,
// so the tensor core works on one tile while the softmax works on the other.
// Every MMA of a tile's chunk is a 128 x 128 x 16 (or 128 x D x 16) step,
// the shape at which the tensor core runs at full rate.
// Ordering facts the protocol relies on (tcgen05 operations issued by one
// thread execute in issue order, and a commit covers all earlier ones):
//  - S_t(j+1) is issued after PV_t(j), so it never overwrites P_t(j) early;
//  - once S_t(j) is complete, so is PV_t(j-1): the softmax may rescale O_t
//    at chunk j without waiting for anything else.
// Every MMA covers a whole chunk, also for the short last chunk of an item:
// the softmax masks the columns past its end (P = 0 there) and the V ring is
// zeroed once at the start, so the stale V rows behind them are finite.
//
// A persistent grid of one CTA per SM takes items dynamically: the TMA warp
// draws the next item index from a global counter and publishes it in a small
// shared-memory ring that every other role reads in the same order.  An item
// of at most 128 query rows splits its key stream between the two tiles (even
// and odd chunks, see plan_item) and merges the two partial softmax results in
// the epilogue.
//
// The softmax splits its exponentials between the special-function unit
// (ex2.approx) and the FMA pipe (2^x = 2^n 2^f, n = rint(x), f in [-1/2, 1/2],
// 2^f by a cubic; Cody and Waite's argument reduction with a polynomial of
// our own fit): at 128 keys per chunk the special-function unit alone would
// take as long per chunk as the tensor core.
// Every mbarrier wait is bounded; on expiry the CTA records ST_TIMEOUT,
// drains its copies and MMAs, frees TMEM and returns.
#include "ac_kernels.cuh"

namespace ac {

template <int D> struct A3Cfg {
    static constexpr int BM = 128, BN = ATTN3_CHUNK, DB = D / 64, KSTEP = 16;
    static constexpr int Q_BYTES = BM * D * 2;     // one query tile
    static constexpr int KV_BYTES = BN * D * 2;    // one stage of K (or of V)
    static constexpr int KST = D == 128 ? 3 : 4, VST = D == 128 ? 2 : 4;
    static constexpr int OFF_Q = 0;                // tile 1 at + Q_BYTES
    static constexpr int OFF_K = 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
    static constexpr int OFF_X = OFF_BAR + 512;    // split items: (max, sum) of tile 1 per row
    static constexpr int OFF_SCHED = OFF_X + 128 * 8;  // ring of scheduled item indices
    static constexpr int SCHED = 4;                // its depth
    static constexpr int SMEM_RAW = OFF_SCHED + 16 * SCHED + 1024;
    // threads that read each ring entry: V producer warp, MMA warp, both softmax warpgroups
    static constexpr int SCHED_READERS = 32 + 32 + 256;
    // at least 116 KB so that two CTAs never share an SM (each takes all of TMEM)
    static constexpr int SMEM = SMEM_RAW > 116 * 1024 ? SMEM_RAW : 116 * 1024;
    // warps 0-3 softmax tile 0, 4-7 softmax tile 1, 8 TMA (Q, K), 9 MMA, 10 TMA (V), 11 idle:
    // three full warpgroups, so registers can move between them (setmaxnreg)
    static constexpr int NTHREADS = 384;
    static constexpr int REGS_LAUNCH = 168, REGS_LOW = 136, REGS_HIGH = 184;
    static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= NTHREADS * REGS_LAUNCH, "register split");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int TM_S = 0;                 // + 128 t
    static constexpr int TM_O = 256;               // + D t
    static_assert(TM_O + 2 * D <= (int)TMEM_COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
    // exponentials per 8 key pairs evaluated on the FMA pipe
    static constexpr int EMU_PER8 = 2;
};

struct A3Params {
    int H, N;
    const int32_t *qperm;
    int kk_cap, kq_cap;
    const int2 *runs;      // per (head, query cluster): ascending key-row runs
    const int2 *run_info;  // per (head, query cluster): {runs, chunks}
    const uint2 *masks;    // per (head, query cluster, chunk): valid rows per 8-row group
    int max_chunks;
    const AttnItem *items;
    const int32_t *n_items;
    int *work;             // items handed out so far (zeroed by the work-list builder)
    // per-query selection: [H, max_chunks, N] by the row's position in cluster
    // order, bit g = the row keeps 8-key group g of the chunk (NULL: all rows keep all)
    const uint16_t *rowmask;
    __nv_bfloat16 *out;
    float *lse;
    int *status;
    float scale_log2;
};

// K or V tensor maps of one operand, one per box height (128 ... 8 rows).
struct KVMaps3 {
    CUtensorMap m128, m64, m32, m16, m8;
};

namespace {

constexpr uint32_t kFullMask = 0x88888888u;  // eight groups of 8 valid rows

__device__ __forceinline__ int item_chunks3(const A3Params &p, const AttnItem &it) {
    if (it.a < 0) return (p.N + ATTN3_CHUNK - 1) / ATTN3_CHUNK;
    return p.run_info[(size_t)it.h * p.kq_cap + it.a].y;
}

// How an item maps onto the CTA's two tiles.  More than 128 query rows: both
// tiles, on the same key chunks.  At most 128 rows and two or more chunks: the
// key stream is split, tile 0 takes the even chunks and tile 1 the odd ones,
// both on the same query rows (one Q tile), and the epilogue merges the two
// partial softmax results, so the tensor core still alternates between two
// tiles.  Interleaving (rather than halving) keeps the chunks in stream order,
// so a split item reads the keys in the same order as every other item of the
// head and finds them in L2.  Otherwise: tile 0 alone.
struct ItemPlan {
    int nt;      // tiles active
    int qt;      // query tiles loaded
    bool split;
    int nc0, nc1;  // chunks of tile 0 / tile 1
};
__device__ __forceinline__ ItemPlan plan_item(const AttnItem &it, int nch) {
    ItemPlan pl;
    pl.split = it.q_len <= 128 && nch >= 2;
    pl.qt = it.q_len > 128 ? 2 : 1;
    pl.nt = (it.q_len > 128 || pl.split) ? 2 : 1;
    pl.nc0 = pl.split ? (nch + 1) / 2 : nch;
    pl.nc1 = pl.split ? nch / 2 : (pl.nt > 1 ? nch : 0);
    return pl;
}

// Valid-row counts (4 bits per 8-row group) of 64 rows whose first `rows` are keys.
__device__ __forceinline__ uint32_t prefix_mask64(int rows) {
    rows = rows < 0 ? 0 : (rows > 64 ? 64 : rows);
    const int nf = rows >> 3;
    uint32_t gm = (nf >= 8 ? 0xFFFFFFFFu : ((1u << (4 * nf)) - 1u)) & kFullMask;
    if (rows & 7) gm |= (uint32_t)(rows & 7) << (4 * nf);
    return gm;
}
// Mask of chunk j of an item: from the precomputed table, or, for a dense head
// (one run of all N rows), from the chunk's position.
__device__ __forceinline__ uint2 item_mask3(const A3Params &p, const uint2 *mrow, int j) {
    if (mrow) {
        // volatile: issued where it stands (two chunks ahead of its use),
        // not moved next to the use
        uint2 r;
        asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(mrow + j));
        return r;
    }
    const int left = p.N - j * ATTN3_CHUNK;
    return make_uint2(prefix_mask64(left), prefix_mask64(left - 64));
}

__device__ __forceinline__ void stream_init3(KeyStream &ks, const A3Params &p, const AttnItem &it) {
    if (it.a < 0) {
        ks.init(nullptr, 1, p.N);
    } else {
        const size_t qa = (size_t)it.h * p.kq_cap + it.a;
        ks.init(p.runs + qa * p.kk_cap, p.run_info[qa].x, p.N);
    }
}

__device__ __forceinline__ void drain3(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = gtimer();
    while (!mbar_try_wait(bar, parity) && gtimer() - t0 < 200000000ull) {
    }
}

template <int R> __device__ __forceinline__ void regs_dec3() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R> __device__ __forceinline__ void regs_inc3() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}

__device__ __forceinline__ uint64_t pack2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t r, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for a pair on the FMA pipe.  x is clamped to [-127, 2^22): with
// n = rint(x) (the 1.5 * 2^23 shift puts it in the low mantissa bits of t) and
// f = x - n in [-1/2, 1/2], 2^f = 1 + c1 f + c2 f^2 + c3 f^3 (relative error
// below 1.1e-4 on that interval: the minimax cubic with constant term 1,
// fitted by linear programming on 4001 points), and adding n << 23 to its bits
// scales it by 2^n.  x = -127 gives exactly +0 (f = 0, p = 1, exponent field 0),
// so masked scores (-inf) contribute nothing; x > -127 gives a normal number
// or, below -126, a nonnegative subnormal.
__device__ __forceinline__ void ex2_poly2(float x0, float x1, float &y0, float &y1) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    x0 = fmaxf(x0, -127.f);
    x1 = fmaxf(x1, -127.f);
    const uint64_t x = pack2(x0, x1);
    const uint64_t t = fadd2(x, pack2(kShift, kShift));
    const uint64_t n = fadd2(t, pack2(-kShift, -kShift));
    const uint64_t f = ffma2(n, pack2(-1.f, -1.f), x);
    uint64_t q = ffma2(pack2(0.0550091f, 0.0550091f), f, pack2(0.2422110f, 0.2422110f));
    q = ffma2(q, f, pack2(0.6932829f, 0.6932829f));
    q = ffma2(q, f, pack2(1.f, 1.f));
    float t0, t1, q0, q1;
    unpack2(t, t0, t1);
    unpack2(q, q0, q1);
    y0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
    y1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// `rows` (a multiple of 8, at most 128) rows from global row `grow` into rows
// r0.. of one K or V stage: one box per set bit of `rows`, per 64-column block.
template <int D>
__device__ __forceinline__ void load_rows3(uint32_t ld, unsigned char *stage, int r0, int grow, int rows,
                                           const KVMaps3 &m, uint64_t *bar, uint64_t pol) {
    using C = A3Cfg<D>;
#pragma unroll
    for (int kb = 0; kb < C::DB; kb++) {
        unsigned char *dst = stage + kb * (C::BN * 128);
        int r = r0, g = grow;
        if (rows & 128) { tma_load_2d_hint_p(ld, dst + r * 128, &m.m128, bar, kb * 64, g, pol); r += 128; g += 128; }
        if (rows & 64) { tma_load_2d_hint_p(ld, dst + r * 128, &m.m64, bar, kb * 64, g, pol); r += 64; g += 64; }
        if (rows & 32) { tma_load_2d_hint_p(ld, dst + r * 128, &m.m32, bar, kb * 64, g, pol); r += 32; g += 32; }
        if (rows & 16) { tma_load_2d_hint_p(ld, dst + r * 128, &m.m16, bar, kb * 64, g, pol); r += 16; g += 16; }
        if (rows & 8) tma_load_2d_hint_p(ld, dst + r * 128, &m.m8, bar, kb * 64, g, pol);
    }
}

// The next chunk of the stream into one stage, each piece into its slot;
// returns the rows loaded.
template <int D>
__device__ __forceinline__ int load_chunk3(uint32_t ld, KeyStream &ks, unsigned char *stage, int row_base,
                                           const KVMaps3 &m, uint64_t *bar, uint64_t pol) {
    using C = A3Cfg<D>;
    int fill = 0, start = 0, valid = 0, slot = 0;
    while (fill < C::BN && ks.piece(C::BN - fill, start, valid, slot)) {
        load_rows3<D>(ld, stage, fill, row_base + start, slot, m, bar, pol);
        fill += slot;
    }
    return fill;
}
// Rows of the next chunk (the same pieces as load_chunk3)
__device__ __forceinline__ int chunk_rows3(KeyStream &ks, int cap) {
    int fill = 0, s, v, sl;
    while (fill < cap && ks.piece(cap - fill, s, v, sl)) fill += sl;
    return fill;
}

// S_t = Q_t K^T into TMEM columns d (the 128 keys of one K stage)
template <int D>
__device__ __forceinline__ void issue_s3(uint32_t ld, uint32_t d, uint64_t qdesc_t, uint64_t kdesc_stage) {
    using C = A3Cfg<D>;
    constexpr uint32_t idesc = idesc_make(128, C::BN, 1, false);
    uint64_t a = qdesc_t, b = kdesc_stage;
#pragma unroll
    for (int kb = 0; kb < C::DB; kb++) {
#pragma unroll
        for (int k4 = 0; k4 < 4; k4++) umma_f16_p(ld, d, a + 2 * k4, b + 2 * k4, idesc, (kb | k4) ? 1u : 0u);
        a += (C::BM * 128) >> 4;
        b += (C::BN * 128) >> 4;
    }
}

// O_t (+)= P_t V over the 128 keys of one V stage; P_t is bf16 in TMEM at a0
// (two keys per 32-bit column)
template <int D>
__device__ __forceinline__ void issue_pv3(uint32_t ld, uint32_t d, uint32_t a0, uint64_t vdesc_stage, bool first) {
    using C = A3Cfg<D>;
    constexpr uint32_t idesc = idesc_make(128, D, 1, true);
#pragma unroll
    for (int ks = 0; ks < C::BN / C::KSTEP; ks++)
        umma_ts_f16_p(ld, d, a0 + ks * 8, vdesc_stage + (uint64_t)((ks * C::KSTEP * 128) >> 4), idesc,
                      (!first || ks > 0) ? 1u : 0u);
}

// Scores of rows nv..7 of 8-row group G set to -inf
template <int G> __device__ __forceinline__ void mask_group(uint32_t (&s)[128], uint32_t nv) {
#pragma unroll
    for (int i = 0; i < 8; i++)
        if ((uint32_t)i >= nv) s[8 * G + i] = __float_as_uint(-INFINITY);
}
// The partial groups of one 32-bit mask word (groups B .. B+7): a group is
// partial when bit 3 of its count is clear (count < 8).  Most chunks hold one
// or two partial groups (one per key run that ends inside the chunk), so only
// those are visited; the switch gives each a body with fixed register indices.
template <int B> __device__ __forceinline__ void mask_word(uint32_t (&s)[128], uint32_t w) {
    uint32_t part = ~w & kFullMask;
    while (part) {
        const int g = (__ffs(part) - 1) >> 2;
        part &= part - 1u;
        const uint32_t nv = (w >> (4 * g)) & 15u;
        switch (g) {
            case 0: mask_group<B + 0>(s, nv); break;
            case 1: mask_group<B + 1>(s, nv); break;
            case 2: mask_group<B + 2>(s, nv); break;
            case 3: mask_group<B + 3>(s, nv); break;
            case 4: mask_group<B + 4>(s, nv); break;
            case 5: mask_group<B + 5>(s, nv); break;
            case 6: mask_group<B + 6>(s, nv); break;
            default: mask_group<B + 7>(s, nv); break;
        }
    }
}
// 8 bits (one per 8-key group) to 8 nibbles: 0xF where the bit is set, 0 elsewhere
__device__ __forceinline__ uint32_t nibbles8(uint32_t b) {
    uint32_t x = b & 0xFFu;
    x = (x | (x << 12)) & 0x000F000Fu;
    x = (x | (x << 6)) & 0x03030303u;
    x = (x | (x << 3)) & 0x11111111u;
    return x * 0xFu;
}
__device__ __forceinline__ uint32_t load_rowmask(const A3Params &p, int h, int chunk, int pos) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];"
                 : "=h"(v)
                 : "l"(p.rowmask + ((size_t)h * p.max_chunks + chunk) * p.N + pos));
    return v;
}
// Scores of 8-row groups past their valid count set to -inf (masks: 4 bits a group)
__device__ __forceinline__ void apply_mask(uint32_t (&s)[128], uint2 gm) {
    if (gm.x != kFullMask) mask_word<0>(s, gm.x);
    if (gm.y != kFullMask) mask_word<8>(s, gm.y);
}

// P for key pairs [P0, P0 + NP) of a row: x = s * scale - m (packed), 2^x on
// MUFU or, for EMU of every 8 pairs, on the FMA pipe; bf16 pairs into pk[pair
// - 32 * (pair / 32)], fp32 sums into la (alternating accumulators)
template <int EMU, int P0, int NP>
__device__ __forceinline__ void exp_pairs(const uint32_t (&s)[128], uint32_t (&pk)[32], uint64_t scale2, uint64_t neg2,
                                          uint64_t (&la)[2]) {
#pragma unroll
    for (int i = P0; i < P0 + NP; i++) {
        float x0, x1, e0, e1;
        unpack2(ffma2(pack2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), scale2, neg2), x0, x1);
        if ((i & 7) >= 8 - EMU) {
            ex2_poly2(x0, x1, e0, e1);
        } else {
            e0 = ex2_approx(x0);
            e1 = ex2_approx(x1);
        }
        la[i & 1] = fadd2(la[i & 1], pack2(e0, e1));
        __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
        pk[i & 31] = *reinterpret_cast<uint32_t *>(&b2);
    }
}

}  // namespace

// ROWS: per-query selection (p.rowmask), a separate instance so that the
// default kernel carries none of its registers.
template <int D, bool ROWS>
__global__ void __launch_bounds__(384, 1)
    attn3_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ KVMaps3 mk,
                 const __grid_constant__ KVMaps3 mv, const A3Params p) {
    using C = A3Cfg<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *q_full = bars + 0, *q_empty = bars + 1;
    uint64_t *k_full = bars + 2, *k_empty = k_full + C::KST;          // [KST]
    uint64_t *v_full = k_empty + C::KST, *v_empty = v_full + C::VST;  // [VST]
    uint64_t *s_full = v_empty + C::VST;  // [tile]: one phase per chunk
    uint64_t *p_full = s_full + 2;        // [tile]: one phase per chunk, 128 arrivals
    uint64_t *o_free = p_full + 2;        // [tile], 128 arrivals
    uint64_t *o_done = o_free + 2;        // [tile]: one phase per item, after its last P.V
    uint64_t *xchg = o_done + 2;          // split items: tile 1's (max, sum) written; 128 arrivals
    uint64_t *comb_done = xchg + 1;       // split items: tile 0 has read O_1; 128 arrivals
    uint64_t *sched_full = comb_done + 1;            // [SCHED], 1 arrival
    uint64_t *sched_empty = sched_full + C::SCHED;   // [SCHED], SCHED_READERS arrivals
    uint64_t *drain_bar = sched_empty + C::SCHED;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(drain_bar + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // zero the V ring once: rows of a stage past its chunk's end are read by
    // P.V (with P = 0) and must hold finite values
    for (int i = threadIdx.x; i < C::VST * C::KV_BYTES / 16; i += C::NTHREADS)
        reinterpret_cast<uint4 *>(sm + C::OFF_V)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < C::KST; i++) {
            mbar_init(k_full + i, 1);
            mbar_init(k_empty + i, 1);
        }
        for (int i = 0; i < C::VST; i++) {
            mbar_init(v_full + i, 1);
            mbar_init(v_empty + i, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(s_full + i, 1);
            mbar_init(p_full + i, 128);
            mbar_init(o_free + i, 128);
            mbar_init(o_done + i, 1);
        }
        mbar_init(xchg, 128);
        mbar_init(comb_done, 128);
        for (int i = 0; i < C::SCHED; i++) {
            mbar_init(sched_full + i, 1);
            mbar_init(sched_empty + i, C::SCHED_READERS);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&mk.m128);
        prefetch_tmap(&mk.m64);
        prefetch_tmap(&mk.m32);
        prefetch_tmap(&mk.m16);
        prefetch_tmap(&mk.m8);
        prefetch_tmap(&mv.m128);
        prefetch_tmap(&mv.m64);
        prefetch_tmap(&mv.m32);
        prefetch_tmap(&mv.m16);
        prefetch_tmap(&mv.m8);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = *p.n_items;
    // Items are handed out dynamically: warp 8 takes the next index from the
    // global work counter and publishes it in a shared ring; every other role
    // reads the same sequence from the ring (-1 ends it).  Items stay in head
    // order, so CTAs working at the same time share a head's keys in L2, and a
    // CTA that drew short items simply takes more of them.
    volatile int *sched_ring = reinterpret_cast<volatile int *>(sm + C::OFF_SCHED);
    uint32_t sched_pos = 0;
    // next item for a reading role (whole warp or warpgroup); -2 on abort
    auto next_item = [&]() -> int {
        const int qs = (int)(sched_pos % C::SCHED);
        if (!mbar_wait_warp(sched_full + qs, (sched_pos / C::SCHED) & 1, abort_flag, p.status)) return -2;
        const int item = sched_ring[qs];
        mbar_arrive(sched_empty + qs);
        sched_pos++;
        return item;
    };

    if (warp >= 8) {
    regs_dec3<C::REGS_LOW>();
    if (warp == 8 || warp == 10) {
        // ------------------------------------------------------ TMA producers
        // Warp 8 loads Q and K, warp 10 loads V.  Each runs its loop converged,
        // with identical values in every lane, and one lane issues the copies.
        const bool kq = warp == 8;
        const uint32_t leader = elect_leader();
        // K/V rows are re-read by every query item of the head: keep them in
        // L2; query tiles are read once: let them go first
        const uint64_t pol_keep = l2_policy_evict_last(), pol_stream = l2_policy_evict_first();
        uint64_t *full = kq ? k_full : v_full, *empty = kq ? k_empty : v_empty;
        const int nst = kq ? C::KST : C::VST;
        unsigned char *ring = sm + (kq ? C::OFF_K : C::OFF_V);
        const KVMaps3 &maps = kq ? mk : mv;
        uint32_t qi = 0, nloads = 0;
        int slot = 0;
        uint32_t phase = 0;  // parity of the current pass over the ring
        bool ok = true;
        // the next chunk of stream `ks` into the next slot of the ring
        auto load_next = [&](KeyStream &ks, int row_base) -> bool {
            KeyStream probe = ks;
            const uint32_t bytes = (uint32_t)chunk_rows3(probe, C::BN) * 128u * C::DB;
            // the slot's previous chunk (one pass ago) must be consumed
            if (nloads >= (uint32_t)nst && !mbar_wait_warp(empty + slot, phase ^ 1u, abort_flag, p.status))
                return false;
            mbar_arrive_expect_tx_p(leader, full + slot, bytes);
            load_chunk3<D>(leader, ks, ring + slot * C::KV_BYTES, row_base, maps, full + slot, pol_keep);
            nloads++;
            if (++slot == nst) {
                slot = 0;
                phase ^= 1u;
            }
            return true;
        };
        for (;;) {
            int item;
            if (kq) {
                // take the next item and publish it
                item = 0;
                if (lane == 0) item = atomicAdd(p.work, 1);
                item = __shfl_sync(0xffffffffu, item, 0);
                if (item >= n_items) item = -1;
                const int qs = (int)(sched_pos % C::SCHED);
                if (sched_pos >= (uint32_t)C::SCHED &&
                    !mbar_wait_warp(sched_empty + qs, ((sched_pos / C::SCHED) - 1) & 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    sched_ring[qs] = item;
                    mbar_arrive(sched_full + qs);
                }
                __syncwarp();
                sched_pos++;
            } else {
                item = next_item();
                if (item == -2) { ok = false; break; }
            }
            if (item < 0) break;
            const AttnItem it = p.items[item];
            const int nch = item_chunks3(p, it);
            if (nch == 0) continue;
            const ItemPlan pl = plan_item(it, nch);
            if (kq) {
                if (qi >= 1 && !mbar_wait_warp(q_empty, (qi - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                mbar_arrive_expect_tx_p(leader, q_full, pl.qt * C::Q_BYTES);
                for (int t = 0; t < pl.qt; t++)
                    for (int kb = 0; kb < C::DB; kb++)
                        tma_load_2d_hint_p(leader, sm + C::OFF_Q + t * C::Q_BYTES + kb * (C::BM * 128), &tmQ, q_full,
                                           kb * 64, it.h * p.N + it.q_start + t * 128, pol_stream);
                qi++;
            }
            KeyStream ks;
            stream_init3(ks, p, it);
            const int row_base = it.h * p.N;
            for (int j = 0; j < nch && ok; j++) ok = load_next(ks, row_base);
            if (!ok) break;
        }
        if (!ok) {
            // wait (bounded) for every copy in flight before the CTA exits
            // (slot i last received load i + nst * ((loads - 1 - i) / nst))
            if (kq && qi >= 1) drain3(q_full, (qi - 1) & 1);
            for (uint32_t i = 0; i < (uint32_t)nst && i < nloads; i++)
                drain3(full + i, ((nloads - 1 - i) / (uint32_t)nst) & 1);
        }
    } else if (warp == 9) {
        // --------------------------------------------------------- MMA issuer
        // The whole warp runs this loop with identical values in every lane;
        // each tcgen05 instruction is issued by one lane, elected once.
        const uint32_t leader = elect_leader();
        uint32_t qi = 0;
        int kslot = 0, vslot = 0;
        uint32_t kph = 0, vph = 0;  // ring pass parities
        uint32_t cnt[2] = {0, 0};   // chunks each tile has been through
        uint32_t act[2] = {0, 0};   // items each tile was active in
        bool ok = true;
        // Descriptors are built once; per MMA only the start-address field
        // (16-byte units, bits 0-13) moves by a compile-time offset.  All
        // shared-memory addresses here are < 256 KB, so the field never carries.
        const uint64_t qdesc = sdesc_sw128(smem_u32(sm + C::OFF_Q), 16, 1024);
        const uint64_t kdesc0 = sdesc_sw128(smem_u32(sm + C::OFF_K), 16, 1024);
        const uint64_t vdesc0 = sdesc_make(smem_u32(sm + C::OFF_V), C::BN * 128, 1024, 2u);
        auto k_next = [&]() {
            if (++kslot == C::KST) {
                kslot = 0;
                kph ^= 1u;
            }
        };
        auto v_next = [&]() {
            if (++vslot == C::VST) {
                vslot = 0;
                vph ^= 1u;
            }
        };
        for (;;) {
            const int item = next_item();
            if (item == -2) { ok = false; break; }
            if (item < 0) break;
            const AttnItem it = p.items[item];
            const int nch = item_chunks3(p, it);
            if (nch == 0) continue;
            const ItemPlan pl = plan_item(it, nch);
            const int nt = pl.nt;
            if (!mbar_wait_warp(q_full, qi & 1, abort_flag, p.status)) { ok = false; break; }
            qi++;
            // K/V stages in stream order.  Unsplit: stage j serves chunk j of
            // both tiles.  Split: stage 2j + t serves chunk j of tile t only.
            // A stage is waited for by its first user and released (empty
            // barrier committed) after its last.
            const int nc[2] = {pl.nc0, pl.nc1};
            const uint64_t qd[2] = {qdesc, qdesc + (uint64_t)((pl.qt > 1 ? C::Q_BYTES : 0) >> 4)};
            int k_used = 0;  // stages of K released in this item
            // prologue: S_t(0)
#pragma unroll
            for (int t = 0; t < 2; t++) {
                if (t >= nt) break;
                if (pl.split || t == 0) {
                    if (!mbar_wait_warp(k_full + kslot, kph, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                }
                issue_s3<D>(leader, tmem + C::TM_S + t * 128, qd[t], kdesc0 + (uint64_t)((kslot * C::KV_BYTES) >> 4));
                umma_commit_p(leader, s_full + t);
                if (pl.split || t == nt - 1) {
                    umma_commit_p(leader, k_empty + kslot);
                    k_next();
                    if (++k_used == nch) umma_commit_p(leader, q_empty);
                }
            }
            for (int j = 0; j < pl.nc0 && ok; j++) {
#pragma unroll
                for (int t = 0; t < 2; t++) {
                    if (t >= nt || j >= nc[t]) break;
                    const uint32_t c = cnt[t] + j;
                    if (pl.split || t == 0) {
                        if (!mbar_wait_warp(v_full + vslot, vph, abort_flag, p.status)) { ok = false; break; }
                    }
                    // PV_t(j) once softmax t has written P_t(j)
                    if (!mbar_wait_warp(p_full + t, c & 1, abort_flag, p.status)) { ok = false; break; }
                    if (j == 0 && act[t] >= 1 && !mbar_wait_warp(o_free + t, (act[t] - 1) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv3<D>(leader, tmem + C::TM_O + t * D, tmem + C::TM_S + t * 128,
                                 vdesc0 + (uint64_t)((vslot * C::KV_BYTES) >> 4), j == 0);
                    if (pl.split || t == nt - 1) {
                        umma_commit_p(leader, v_empty + vslot);
                        v_next();
                    }
                    if (j + 1 == nc[t]) {
                        umma_commit_p(leader, o_done + t);
                        continue;
                    }
                    // S_t(j+1) into S_t, behind the P.V that reads P_t(j) from it
                    if (pl.split || t == 0) {
                        if (!mbar_wait_warp(k_full + kslot, kph, abort_flag, p.status)) { ok = false; break; }
                        tc_fence_after();
                    }
                    issue_s3<D>(leader, tmem + C::TM_S + t * 128, qd[t], kdesc0 + (uint64_t)((kslot * C::KV_BYTES) >> 4));
                    umma_commit_p(leader, s_full + t);
                    if (pl.split || t == nt - 1) {
                        umma_commit_p(leader, k_empty + kslot);
                        k_next();
                        if (++k_used == nch) umma_commit_p(leader, q_empty);
                    }
                }
            }
            if (!ok) break;
            cnt[0] += pl.nc0;
            act[0]++;
            if (nt > 1) {
                cnt[1] += pl.nc1;
                act[1]++;
            }
        }
        if (!ok) {
            umma_commit_p(leader, drain_bar);
            drain3(drain_bar, 0);
        }
    }
    // teardown inside each branch (no code after the role split is shared by
    // warps of different register budgets): all 384 threads meet at barrier 1,
    // then the allocating warp frees TMEM
    tc_fence_before();
    named_bar_sync(1, C::NTHREADS);
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    } else {
        regs_inc3<C::REGS_HIGH>();
        // ------------------------------------------------ softmax + epilogue
        // Warpgroup t = tile t; one thread per query row (= TMEM lane).
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_addr = tmem + lane_addr + C::TM_S + t * 128;
        const uint32_t o_addr = tmem + lane_addr + C::TM_O + t * D;
        const float sc = p.scale_log2;
        uint32_t cnt = 0;         // chunks (= s_full / p_full phases) this tile has been through
        uint32_t items_done = 0;  // items (= o_done phases) this tile has finished
        uint32_t splits = 0;      // split items (= xchg / comb_done phases) so far
        float2 *xs = reinterpret_cast<float2 *>(sm + C::OFF_X);
        bool ok = true;
        for (;;) {
            const int item = next_item();
            if (item == -2) { ok = false; break; }
            if (item < 0) break;
            const AttnItem it = p.items[item];
            const int nch_all = item_chunks3(p, it);
            const ItemPlan pl = plan_item(it, nch_all);
            if (t >= pl.nt) continue;
            // this tile's chunk j is chunk cbase + cstep j of the item's key stream
            const int nch = t == 0 ? pl.nc0 : pl.nc1;
            const int cbase = pl.split ? t : 0, cstep = pl.split ? 2 : 1;
            const int r = pl.split ? row : t * 128 + row;
            const bool valid = r < it.q_len;
            int tok = 0;
            if (valid) tok = p.qperm[(size_t)it.h * p.N + it.q_start + r];
            __nv_bfloat16 *orow = p.out + ((size_t)it.h * p.N + tok) * D;
            if (nch == 0) {
                if (valid) {
                    for (int k = 0; k < D; k++) orow[k] = __float2bfloat16(0.f);
                    if (p.lse) p.lse[(size_t)it.h * p.N + tok] = -INFINITY;
                }
                continue;
            }
            // valid rows per 8-row group of each chunk (4 bits each, 8 = all),
            // precomputed from the key runs; the next chunk's mask is loaded ahead
            const uint2 *mrow = it.a < 0 ? nullptr : p.masks + ((size_t)it.h * p.kq_cap + it.a) * p.max_chunks;
            // masks are fetched two chunks ahead, so the load has a whole
            // chunk's time to arrive before its value is needed
            uint2 gm_next = item_mask3(p, mrow, cbase);
            uint2 gm_next2 = nch > 1 ? item_mask3(p, mrow, cbase + cstep) : make_uint2(0u, 0u);
            // per-query selection: the row's own groups of each chunk, also two ahead
            const bool own = ROWS && it.a >= 0 && valid;
            const int rpos = it.q_start + r;
            uint32_t rm_next = own ? load_rowmask(p, it.h, cbase, rpos) : 0xFFFFu;
            uint32_t rm_next2 = own && nch > 1 ? load_rowmask(p, it.h, cbase + cstep, rpos) : 0xFFFFu;
            float m_ref = -INFINITY, l0 = 0.f, l1 = 0.f;
            for (int j = 0; j < nch; j++) {
                uint2 gm = gm_next;
                gm_next = gm_next2;
                if (j + 2 < nch) gm_next2 = item_mask3(p, mrow, cbase + cstep * (j + 2));
                uint32_t drop = 0u;  // per-query selection: 8-key groups this row does not keep
                if (ROWS) {
                    const uint32_t rm = rm_next;
                    rm_next = rm_next2;
                    if (own && j + 2 < nch) rm_next2 = load_rowmask(p, it.h, cbase + cstep * (j + 2), rpos);
                    drop = ~rm & 0xFFFFu;
                }
                const uint32_t c = cnt + j;
                if (!mbar_wait_warp(s_full + t, c & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                // Per-query selection: a warp none of whose rows takes a key of
                // this chunk (rows that keep none of the chunk's groups, and rows
                // past the item's query rows, whose output is never written)
                // would compute P = 0 with its row maxima, sums and O unchanged:
                // it stores the zeros (after S_t(j) is complete, as P always is)
                // and skips the rest.  (The default instance gained nothing from
                // skipping its all-padding warps and keeps the full path.)
                if (ROWS && __all_sync(0xffffffffu, !valid || drop == 0xFFFFu)) {
                    tmem_st32_zero(s_addr);
                    tmem_st32_zero(s_addr + 32);
                } else {
                    uint32_t s[128];
                    tmem_ld128(s_addr, s);
                    apply_mask(s, gm);
                    if (ROWS && drop) {
                        // a row keeps about one group in seven of its tile's union:
                        // every group is dropped by predicated selects, not visited
                        // one by one as the chunk's few partial groups are
#pragma unroll
                        for (int g = 0; g < 16; g++) {
                            const bool d = (drop >> g) & 1u;
#pragma unroll
                            for (int i = 0; i < 8; i++) s[8 * g + i] = d ? __float_as_uint(-INFINITY) : s[8 * g + i];
                        }
                    }
                    // row max: four independent chains of 3-input max
                    float mq[4];
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        float m = fmaxf(__uint_as_float(s[32 * q]), __uint_as_float(s[32 * q + 1]));
#pragma unroll
                        for (int i = 2; i < 32; i += 2)
                            m = fmax3(m, __uint_as_float(s[32 * q + i]), __uint_as_float(s[32 * q + i + 1]));
                        mq[q] = m;
                    }
                    const float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
                    const float m_new = mx * sc;
                    if (j == 0) m_ref = m_new;
                    // Move the reference max (and rescale O_t and l by f) only when it
                    // grew by more than 2^8; warp-uniform because TMEM access is
                    // collective.  The rescale of O_t waits until P_t(j) is stored (the
                    // scores are then dead, which keeps the register peak low); it
                    // only has to precede the arrival that lets PV_t(j) go, and
                    // PV_t(j-1) is complete: S_t(j) was issued after it.
                    const bool rescale = j > 0 && __any_sync(0xffffffffu, m_new > m_ref + 8.f);
                    float f = 1.f;
                    if (rescale) {
                        const float m_to = fmaxf(m_ref, m_new);
                        // a row with no unmasked key yet keeps f = 1 (its O and l are 0)
                        f = m_to == -INFINITY ? 1.f : ex2_approx(m_ref - m_to);
                        m_ref = m_to;
                    }
                    // a row whose keys so far are all masked (per-query selection) has
                    // m_ref = -inf: its scores are all -inf and must give P = 0
                    const float negm = m_ref == -INFINITY ? 0.f : -m_ref;
                    const uint64_t scale2 = pack2(sc, sc), neg2 = pack2(negm, negm);
                    // row sum in four partial sums (two packed pairs), folded into l0/l1
                    uint64_t la[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
                    uint32_t pk[32];
                    exp_pairs<C::EMU_PER8, 0, 32>(s, pk, scale2, neg2, la);
                    tmem_st32(s_addr, pk);
                    exp_pairs<C::EMU_PER8, 32, 32>(s, pk, scale2, neg2, la);
                    tmem_st32(s_addr + 32, pk);
                    if (rescale) {
#pragma unroll
                        for (int pc = 0; pc < D / 32; pc++) {
                            uint32_t o[32];
                            tmem_ld32(o_addr + pc * 32, o);
#pragma unroll
                            for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                            tmem_st32(o_addr + pc * 32, o);
                        }
                    }
                    float a0, a1, b0, b1;
                    unpack2(la[0], a0, a1);
                    unpack2(la[1], b0, b1);
                    l0 = fmaf(l0, f, a0 + b0);
                    l1 = fmaf(l1, f, a1 + b1);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_full + t);
            }
            if (!ok) break;
            if (pl.split) {
                // Split item.  Tile 1 hands its row max and sum to tile 0 through
                // shared memory; tile 0 merges O_0 and O_1 (both in TMEM, same
                // lanes) with weights 2^(m_t - m), m = max(m_0, m_1), and writes
                // the rows.  Tile 1 releases O_1 only once tile 0 has read it.
                if (!mbar_wait_warp(o_done + t, items_done & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                if (t == 1) {
                    xs[row] = make_float2(m_ref, l0 + l1);
                    tc_fence_before();  // O_1 is final (o_done); tile 0 reads it after xchg
                    mbar_arrive(xchg);
                    if (!mbar_wait_warp(comb_done, splits & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    tc_fence_before();
                    mbar_arrive(o_free + 1);
                } else {
                    if (!mbar_wait_warp(xchg, splits & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const float2 x1 = xs[row];
                    const float m = fmaxf(m_ref, x1.x);
                    const float w0 = ex2_approx(m_ref - m), w1 = ex2_approx(x1.x - m);
                    const float lsum = (l0 + l1) * w0 + x1.y * w1;
                    const float inv = 1.f / lsum;
                    const float a0 = w0 * inv, a1 = w1 * inv;
#pragma unroll
                    for (int pc = 0; pc < D / 32; pc++) {
                        uint32_t o[32], o1[32];
                        tmem_ld32(o_addr + pc * 32, o);
                        tmem_ld32(o_addr + D + pc * 32, o1);
                        if (valid) {
                            uint32_t w[16];
#pragma unroll
                            for (int i = 0; i < 16; i++) {
                                const float v0 = __uint_as_float(o[2 * i]) * a0 + __uint_as_float(o1[2 * i]) * a1;
                                const float v1 =
                                    __uint_as_float(o[2 * i + 1]) * a0 + __uint_as_float(o1[2 * i + 1]) * a1;
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
                                w[i] = *reinterpret_cast<uint32_t *>(&b2);
                            }
                            uint4 *dst = reinterpret_cast<uint4 *>(orow + pc * 32);
#pragma unroll
                            for (int i = 0; i < 4; i++)
                                __stcs(dst + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(comb_done);
                    mbar_arrive(o_free + 0);
                    if (valid && p.lse) p.lse[(size_t)it.h * p.N + tok] = (m + __log2f(lsum)) * 0.69314718055994531f;
                }
                cnt += nch;
                items_done++;
                splits++;
                continue;
            }
            // epilogue: O_t / l once the last P.V is done, rows scattered back to
            // token order
            if (!mbar_wait_warp(o_done + t, items_done & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            const float lsum = l0 + l1;
            const float inv = 1.f / lsum;
#pragma unroll
            for (int pc = 0; pc < D / 32; pc++) {
                uint32_t o[32];
                tmem_ld32(o_addr + pc * 32, o);
                if (valid) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
                        w[i] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + pc * 32);
#pragma unroll
                    for (int i = 0; i < 4; i++) __stcs(dst + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(o_free + t);
            if (valid && p.lse) p.lse[(size_t)it.h * p.N + tok] = (m_ref + __log2f(lsum)) * 0.69314718055994531f;
            cnt += nch;
            items_done++;
        }
        tc_fence_before();
        named_bar_sync(1, C::NTHREADS);
    }
}

typedef CUresult (*EncodeTiledFn3)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static int bf16_map3(EncodeTiledFn3 enc, CUtensorMap *m, const void *base, int rows, int cols, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
               ? 0
               : -1;
}

static int kv_maps3(EncodeTiledFn3 enc, KVMaps3 *m, const void *base, int rows, int cols) {
    return (bf16_map3(enc, &m->m128, base, rows, cols, 128) || bf16_map3(enc, &m->m64, base, rows, cols, 64) ||
            bf16_map3(enc, &m->m32, base, rows, cols, 32) || bf16_map3(enc, &m->m16, base, rows, cols, 16) ||
            bf16_map3(enc, &m->m8, base, rows, cols, 8))
               ? -1
               : 0;
}

template <int D, bool ROWS>
static int launch3(const void *qg, const void *kg, const void *vg, const A3Params &p, int max_items, int num_sms,
                   void *encode_fn, cudaStream_t st) {
    using C = A3Cfg<D>;
    EncodeTiledFn3 enc = (EncodeTiledFn3)encode_fn;
    CUtensorMap mq;
    KVMaps3 mk, mv;
    const int rows = p.H * p.N;
    if (bf16_map3(enc, &mq, qg, rows, D, 128) || kv_maps3(enc, &mk, kg, rows, D) || kv_maps3(enc, &mv, vg, rows, D))
        return -1;
    // the register split assumes the launch budget ptxas gave the kernel; a
    // larger split would make setmaxnreg.inc wait forever, so refuse.  The
    // shared-memory attribute belongs to the current device: set on every call.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn3_kernel<D, ROWS>) != cudaSuccess || fa.numRegs != C::REGS_LAUNCH) return -1;
    if (cudaFuncSetAttribute(attn3_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return -1;
    int grid = max_items < num_sms ? max_items : num_sms;
    if (grid < 1) grid = 1;
    attn3_kernel<D, ROWS><<<grid, C::NTHREADS, C::SMEM, st>>>(mq, mk, mv, p);
    note_launch();
    return 0;
}

int k_attention3(int D, int H, int N, const void *qg, const void *kg, const void *vg, const int32_t *qperm,
                 int kk_cap, int kq_cap, const int2 *runs, const int2 *run_info, const uint32_t *masks,
                 int max_chunks, const AttnItem *items, const int32_t *n_items, int max_items, void *out, float *lse,
                 int *status, int num_sms, void *encode_fn, cudaStream_t st, const uint16_t *rowmask) {
    A3Params p;
    p.H = H;
    p.N = N;
    p.qperm = qperm;
    p.kk_cap = kk_cap;
    p.kq_cap = kq_cap;
    p.runs = runs;
    p.run_info = run_info;
    p.masks = reinterpret_cast<const uint2 *>(masks);
    p.max_chunks = max_chunks;
    p.items = items;
    p.n_items = n_items;
    p.work = const_cast<int32_t *>(n_items) + 1;
    p.out = reinterpret_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = status;
    p.rowmask = rowmask;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    if (rowmask) {
        if (D == 64) return launch3<64, true>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
        return launch3<128, true>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
    }
    if (D == 64) return launch3<64, false>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
    return launch3<128, false>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
}

}  // namespace ac
