// Block-sparse exact softmax attention over selected key clusters (AdaCluster,
// Algorithm 3 line 9; line 4 for dense heads), bf16 inputs, two query tiles
// per CTA.
//
// A work item is up to 256 query rows of one query cluster (two 128-row
// tiles) that share one key stream (KeyStream): the rows of the cluster's key
// runs packed into chunks of 64 keys, loaded by TMA into 4-stage K and V rings.
// Each tile owns two S buffers in TMEM, so while softmax warpgroup t turns
// S_t(j) into P_t(j) (bf16, written back over the same columns) the tensor
// core already computes S_t(j+1) in the other buffer.  The single MMA thread
// issues, per chunk j,
//   O_t += P_t(j) V_j          (A operand read from TMEM) once P_t(j) is written, t = 0, 1,
//   S_t(j+2) = Q_t K_{j+2}^T   into the buffer that P_t(j) occupied, t = 0, 1.
// Ordering facts the protocol relies on (tcgen05 operations issued by one
// thread execute in issue order, and a commit covers all earlier ones):
//  - S_t(j+2) is issued after PV_t(j), so it never overwrites P_t(j) early;
//  - once S_t(j) is complete, so is PV_t(j-2), the last reader of its buffer;
//  - PV_t(j-1) may still run while the softmax works on chunk j, so before it
//    rescales O_t the softmax waits for the P.V barrier phase of chunk j-1.
// Every MMA covers a whole 64-key chunk, also for the short last chunk of an
// item: the softmax masks the columns past its end (P = 0 there) and the V
// ring is zeroed once at the start, so the stale K/V rows behind them are
// finite.  A runtime guard per MMA instruction made the issue about 2.5x
// slower on B200, and the MMA warp then needs no chunk sizes at all.
// Every mbarrier wait is bounded; on expiry the CTA records ST_TIMEOUT,
// drains its copies and MMAs, frees TMEM and returns.
#include "ac_kernels.cuh"

namespace ac {

template <int D> struct A2Cfg {
    static constexpr int BM = 128, BN = ATTN2_CHUNK, DB = D / 64, KSTEP = 16;
    static constexpr int Q_BYTES = BM * D * 2;     // one query tile
    static constexpr int KV_BYTES = BN * D * 2;    // one stage of K (or of V)
    static constexpr int KST = 4, VST = 4;
    static constexpr int OFF_Q = 0;                // tile 1 at + Q_BYTES
    static constexpr int OFF_K = 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
    static constexpr int SMEM_RAW = OFF_BAR + 512 + 1024;
    // at least 116 KB so that two CTAs never share an SM (each takes all of TMEM)
    static constexpr int SMEM = SMEM_RAW > 116 * 1024 ? SMEM_RAW : 116 * 1024;
    // warps 0-3 softmax tile 0, 4-7 softmax tile 1, 8 TMA (Q, K), 9 MMA, 10 TMA (V), 11 idle:
    // three full warpgroups, so registers can move between them (setmaxnreg)
    static constexpr int NTHREADS = 384;
    static constexpr int REGS_LAUNCH = 168, REGS_LOW = 152, REGS_HIGH = 176;
    static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= NTHREADS * REGS_LAUNCH, "register split");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int TM_S = 0;                 // + 128 t + 64 buffer
    static constexpr int TM_O = 256;               // + D t
    static_assert(TM_O + 2 * D <= (int)TMEM_COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct A2Params {
    int H, N;
    const int32_t *qperm;
    int kk_cap, kq_cap;
    const int2 *runs;      // per (head, query cluster): ascending key-row runs
    const int2 *run_info;  // per (head, query cluster): {runs, chunks}
    const uint32_t *masks; // per (head, query cluster, chunk): valid rows per 8-row group
    int max_chunks;
    const AttnItem *items;
    const int32_t *n_items;
    __nv_bfloat16 *out;
    float *lse;
    int *status;
    float scale_log2;
};

// K or V tensor maps of one operand, one per box height (64, 32, 16, 8 rows).
struct KVMaps {
    CUtensorMap m64, m32, m16, m8;
};

namespace {

__device__ __forceinline__ int item_chunks(const A2Params &p, const AttnItem &it) {
    if (it.a < 0) return (p.N + ATTN2_CHUNK - 1) / ATTN2_CHUNK;
    return p.run_info[(size_t)it.h * p.kq_cap + it.a].y;
}

// Valid-row counts (4 bits per 8-row group) of a chunk whose first `rows` rows are keys.
__device__ __forceinline__ uint32_t prefix_mask(int rows) {
    const int nf = rows >> 3;
    uint32_t gm = (nf >= 8 ? 0xFFFFFFFFu : ((1u << (4 * nf)) - 1u)) & 0x88888888u;
    if (rows & 7) gm |= (uint32_t)(rows & 7) << (4 * nf);
    return gm;
}
// Mask of chunk j of an item: from the precomputed table, or, for a dense head
// (one run of all N rows), from the chunk's position.
__device__ __forceinline__ uint32_t item_mask(const A2Params &p, const uint32_t *mrow, int j) {
    if (mrow) return __ldg(mrow + j);
    const int left = p.N - j * ATTN2_CHUNK;
    return prefix_mask(left > ATTN2_CHUNK ? ATTN2_CHUNK : left);
}

__device__ __forceinline__ void stream_init(KeyStream &ks, const A2Params &p, const AttnItem &it) {
    if (it.a < 0) {
        ks.init(nullptr, 1, p.N);
    } else {
        const size_t qa = (size_t)it.h * p.kq_cap + it.a;
        ks.init(p.runs + qa * p.kk_cap, p.run_info[qa].x, p.N);
    }
}

__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *status) {
    return mbar_wait_warp(bar, parity, abort_flag, status);
}

__device__ __forceinline__ void drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = gtimer();
    while (!mbar_try_wait(bar, parity) && gtimer() - t0 < 200000000ull) {
    }
}

template <int R> __device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R> __device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}

// (a0, a1) * s + c, two lanes of one packed fp32 FMA
__device__ __forceinline__ void fma2(float &o0, float &o1, float a0, float a1, float s, float c) {
    uint64_t a, b, d, e;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %1};" : "=l"(b) : "f"(s));
    asm("mov.b64 %0, {%1, %1};" : "=l"(e) : "f"(c));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(e));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(o0), "=f"(o1) : "l"(d));
}

// (a0, a1) + (b0, b1), one packed fp32 add
__device__ __forceinline__ void add2(float &a0, float &a1, float b0, float b1) {
    uint64_t a, b, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(d));
}

// `rows` (a multiple of 8, at most 64) rows from global row `grow` into rows
// r0.. of one K or V stage: one box per set bit of `rows`, per 64-column block.
template <int D>
__device__ __forceinline__ void load_rows(uint32_t ld, unsigned char *stage, int r0, int grow, int rows,
                                          const KVMaps &m, uint64_t *bar, uint64_t pol) {
    using C = A2Cfg<D>;
#pragma unroll
    for (int kb = 0; kb < C::DB; kb++) {
        unsigned char *dst = stage + kb * (C::BN * 128);
        int r = r0, g = grow;
        if (rows & 64) { tma_load_2d_hint_p(ld, dst + r * 128, &m.m64, bar, kb * 64, g, pol); r += 64; g += 64; }
        if (rows & 32) { tma_load_2d_hint_p(ld, dst + r * 128, &m.m32, bar, kb * 64, g, pol); r += 32; g += 32; }
        if (rows & 16) { tma_load_2d_hint_p(ld, dst + r * 128, &m.m16, bar, kb * 64, g, pol); r += 16; g += 16; }
        if (rows & 8) tma_load_2d_hint_p(ld, dst + r * 128, &m.m8, bar, kb * 64, g, pol);
    }
}

// The next chunk of the stream into one stage, each piece into its slot;
// returns the rows loaded.
template <int D>
__device__ __forceinline__ int load_chunk(uint32_t ld, KeyStream &ks, unsigned char *stage, int row_base,
                                          const KVMaps &m, uint64_t *bar, uint64_t pol) {
    using C = A2Cfg<D>;
    int fill = 0, start = 0, valid = 0, slot = 0;
    while (fill < C::BN && ks.piece(C::BN - fill, start, valid, slot)) {
        load_rows<D>(ld, stage, fill, row_base + start, slot, m, bar, pol);
        fill += slot;
    }
    return fill;
}
// Rows of the next chunk (the same pieces as load_chunk)
__device__ __forceinline__ int chunk_rows(KeyStream &ks, int cap) {
    int fill = 0, s, v, sl;
    while (fill < cap && ks.piece(cap - fill, s, v, sl)) fill += sl;
    return fill;
}

// S_t = Q_t K^T into TMEM columns d (the 64 keys of one K stage); whole warp
template <int D>
__device__ __forceinline__ void issue_s(uint32_t ld, uint32_t d, uint64_t qdesc_t, uint64_t kdesc_stage) {
    using C = A2Cfg<D>;
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

// O_t (+)= P_t V over the 64 keys of one V stage; P_t is bf16 in TMEM at a0
// (two keys per 32-bit column); whole warp
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t ld, uint32_t d, uint32_t a0, uint64_t vdesc_stage, bool first) {
    using C = A2Cfg<D>;
    constexpr uint32_t idesc = idesc_make(128, D, 1, true);
#pragma unroll
    for (int ks = 0; ks < C::BN / C::KSTEP; ks++)
        umma_ts_f16_p(ld, d, a0 + ks * 8, vdesc_stage + (uint64_t)((ks * C::KSTEP * 128) >> 4), idesc,
                      (!first || ks > 0) ? 1u : 0u);
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ KVMaps mk,
                 const __grid_constant__ KVMaps mv, const A2Params p) {
    using C = A2Cfg<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint64_t *q_full = bars + 0, *q_empty = bars + 1;
    uint64_t *k_full = bars + 2, *k_empty = k_full + C::KST;   // [KST]
    uint64_t *v_full = k_empty + C::KST, *v_empty = v_full + C::VST;  // [VST]
    uint64_t *s_full = v_empty + C::VST;    // [tile][buffer]
    uint64_t *p_full = s_full + 4;          // [tile][buffer], 128 arrivals
    uint64_t *pv_bar = p_full + 4;          // [tile]: one phase per P.V
    uint64_t *o_free = pv_bar + 2;          // [tile], 128 arrivals
    uint64_t *o_done = o_free + 2;          // [tile]: one phase per item, after its last P.V
    uint64_t *drain_bar = o_done + 2;
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
        for (int i = 0; i < 4; i++) {
            mbar_init(s_full + i, 1);
            mbar_init(p_full + i, 128);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(pv_bar + i, 1);
            mbar_init(o_free + i, 128);
            mbar_init(o_done + i, 1);
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
        prefetch_tmap(&mk.m64);
        prefetch_tmap(&mk.m32);
        prefetch_tmap(&mk.m16);
        prefetch_tmap(&mk.m8);
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

    if (warp >= 8) {
    regs_dec<C::REGS_LOW>();
    if (warp == 8 || warp == 10) {
        // ------------------------------------------------------ TMA producers
        // Warp 8 loads Q and K, warp 10 loads V.  Each runs its loop converged,
        // with identical values in every lane, and one lane issues the copies.
        // One lone thread loading K and V in turn could not keep up: the V
        // ring frees slots late (after P.V), and each K load waited behind it.
        const bool kq = warp == 8;
        const uint32_t leader = elect_leader();
        // K/V rows are re-read by every query item of the head: keep them in
        // L2; query tiles are read once: let them go first
        const uint64_t pol_keep = l2_policy_evict_last(), pol_stream = l2_policy_evict_first();
        uint64_t *full = kq ? k_full : v_full, *empty = kq ? k_empty : v_empty;
        constexpr int NST = C::KST;  // == C::VST
        static_assert(C::KST == C::VST, "one ring depth for both producers");
        unsigned char *ring = sm + (kq ? C::OFF_K : C::OFF_V);
        const KVMaps &maps = kq ? mk : mv;
        uint32_t g = 0, qi = 0, nloads = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const AttnItem it = p.items[item];
            const int nch = item_chunks(p, it);
            if (nch == 0) continue;
            if (kq) {
                const int nt = it.q_len > 128 ? 2 : 1;
                if (qi >= 1 && !mbar_wait_warp(q_empty, (qi - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                mbar_arrive_expect_tx_p(leader, q_full, nt * C::Q_BYTES);
                for (int t = 0; t < nt; t++)
                    for (int kb = 0; kb < C::DB; kb++)
                        tma_load_2d_hint_p(leader, sm + C::OFF_Q + t * C::Q_BYTES + kb * (C::BM * 128), &tmQ, q_full,
                                           kb * 64, it.h * p.N + it.q_start + t * 128, pol_stream);
                qi++;
            }
            KeyStream ks;
            stream_init(ks, p, it);
            const int row_base = it.h * p.N;
            for (int j = 0; j < nch; j++, g++) {
                KeyStream probe = ks;
                const uint32_t bytes = (uint32_t)chunk_rows(probe, C::BN) * 128u * C::DB;
                const int slot = g % NST;
                const uint32_t u = g / NST;
                if (u >= 1 && !mbar_wait_warp(empty + slot, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                mbar_arrive_expect_tx_p(leader, full + slot, bytes);
                load_chunk<D>(leader, ks, ring + slot * C::KV_BYTES, row_base, maps, full + slot, pol_keep);
                nloads = g + 1;
            }
        }
        if (!ok) {
            // wait (bounded) for every copy in flight before the CTA exits
            // (slot i last received chunk i + NST * ((loads - 1 - i) / NST))
            if (kq && qi >= 1) drain(q_full, (qi - 1) & 1);
            for (uint32_t i = 0; i < (uint32_t)NST && i < nloads; i++) drain(full + i, ((nloads - 1 - i) / NST) & 1);
        }
    } else if (warp == 9) {
        // --------------------------------------------------------- MMA issuer
        // The whole warp runs this loop with identical values in every lane;
        // each tcgen05 instruction is issued by one elected lane.
        {
            // the lane that issues every tcgen05 instruction, chosen once
            const uint32_t leader = elect_leader();
            uint32_t g = 0, qi = 0;
            uint32_t cnt[2] = {0, 0};  // chunks each tile has been through
            uint32_t act[2] = {0, 0};  // items each tile was active in
            bool ok = true;
            // Descriptors are built once; per MMA only the start-address field
            // (16-byte units, bits 0-13) moves by a compile-time offset.  All
            // shared-memory addresses here are < 256 KB, so the field never carries.
            const uint64_t qdesc = sdesc_sw128(smem_u32(sm + C::OFF_Q), 16, 1024);
            const uint64_t kdesc0 = sdesc_sw128(smem_u32(sm + C::OFF_K), 16, 1024);
            const uint64_t vdesc0 = sdesc_make(smem_u32(sm + C::OFF_V), C::BN * 128, 1024, 2u);
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                const AttnItem it = p.items[item];
                const int nch = item_chunks(p, it);
                if (nch == 0) continue;
                const int nt = it.q_len > 128 ? 2 : 1;
                if (!wait_warp(q_full, qi & 1, abort_flag, p.status)) { ok = false; break; }
                qi++;
                // prologue: S_t(0) and S_t(1)
                for (int jj = 0; jj < 2 && jj < nch && ok; jj++) {
                    const uint32_t gk = g + jj;
                    const int kslot = gk % C::KST;
                    if (!wait_warp(k_full + kslot, (gk / C::KST) & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int t = 0; t < 2; t++) {
                        if (t >= nt) break;
                        const int b = (cnt[t] + jj) & 1;
                        issue_s<D>(leader, tmem + C::TM_S + t * 128 + b * 64, qdesc + (uint64_t)((t * C::Q_BYTES) >> 4),
                                   kdesc0 + (uint64_t)((kslot * C::KV_BYTES) >> 4));
                        umma_commit_p(leader, s_full + 2 * t + b);
                    }
                    umma_commit_p(leader, k_empty + kslot);
                }
                if (!ok) break;
                if (nch <= 2) umma_commit_p(leader, q_empty);
                for (int j = 0; j < nch && ok; j++) {
                    const uint32_t gv = g + j;
                    const int vslot = gv % C::VST;
                    if (!wait_warp(v_full + vslot, (gv / C::VST) & 1, abort_flag, p.status)) { ok = false; break; }
                    const bool more = j + 2 < nch;
                    const uint32_t gk = g + j + 2;
                    const int kslot = gk % C::KST;
#pragma unroll
                    for (int t = 0; t < 2; t++) {
                        if (t >= nt) break;
                        const uint32_t c = cnt[t] + j;
                        const int b = c & 1;
                        // PV_t(j) once softmax t has written P_t(j)
                        if (!wait_warp(p_full + 2 * t + b, (c >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                        if (j == 0 && act[t] >= 1 && !wait_warp(o_free + t, (act[t] - 1) & 1, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_pv<D>(leader, tmem + C::TM_O + t * D, tmem + C::TM_S + t * 128 + b * 64,
                                    vdesc0 + (uint64_t)((vslot * C::KV_BYTES) >> 4), j == 0);
                        umma_commit_p(leader, pv_bar + t);
                    }
                    // S_t(j+2) into the buffers P_t(j) occupied, after both P.V
                    // groups: the other tile's P.V runs between the reads of a
                    // buffer and its overwrite
                    if (ok && more) {
                        if (!wait_warp(k_full + kslot, (gk / C::KST) & 1, abort_flag, p.status)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int t = 0; t < 2; t++) {
                            if (t >= nt) break;
                            const int b = (cnt[t] + j) & 1;
                            issue_s<D>(leader, tmem + C::TM_S + t * 128 + b * 64, qdesc + (uint64_t)((t * C::Q_BYTES) >> 4),
                                       kdesc0 + (uint64_t)((kslot * C::KV_BYTES) >> 4));
                            umma_commit_p(leader, s_full + 2 * t + b);
                        }
                    }
                    if (!ok) break;
                    umma_commit_p(leader, v_empty + vslot);
                    if (more) {
                        umma_commit_p(leader, k_empty + kslot);
                        if (j + 3 == nch) umma_commit_p(leader, q_empty);
                    }
                }
                if (!ok) break;
                // the item's last P.V of each tile is done once these arrive
                umma_commit_p(leader, o_done + 0);
                if (nt > 1) umma_commit_p(leader, o_done + 1);
                g += nch;
                cnt[0] += nch;
                act[0]++;
                if (nt > 1) {
                    cnt[1] += nch;
                    act[1]++;
                }
            }
            if (!ok) {
                umma_commit_p(leader, drain_bar);
                drain(drain_bar, 0);
            }
        }
    }
    } else {
        regs_inc<C::REGS_HIGH>();
        // ------------------------------------------------ softmax + epilogue
        // Warpgroup t = tile t; one thread per query row (= TMEM lane).
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t s_base = tmem + lane_addr + C::TM_S + t * 128;
        const uint32_t o_addr = tmem + lane_addr + C::TM_O + t * D;
        const float sc = p.scale_log2;
        uint32_t cnt = 0;         // chunks (= pv_bar phases) this tile has been through
        uint32_t items_done = 0;  // items (= o_done phases) this tile has finished
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const AttnItem it = p.items[item];
            const int nt = it.q_len > 128 ? 2 : 1;
            if (t >= nt) continue;
            const int nch = item_chunks(p, it);
            const int r = t * 128 + row;
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
            // valid rows per 8-row group of each chunk, 4 bits each (8 = all),
            // precomputed from the key runs; the next chunk's mask is loaded ahead
            const uint32_t *mrow = it.a < 0 ? nullptr : p.masks + ((size_t)it.h * p.kq_cap + it.a) * p.max_chunks;
            uint32_t gm_next = item_mask(p, mrow, 0);
            float m_ref = -INFINITY, l0 = 0.f, l1 = 0.f;
            for (int j = 0; j < nch; j++) {
                const uint32_t gm = gm_next;
                if (j + 1 < nch) gm_next = item_mask(p, mrow, j + 1);
                const uint32_t c = cnt + j;
                const int b = c & 1;
                if (!wait_warp(s_full + 2 * t + b, (c >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                uint32_t s[64];
                tmem_ld64(s_base + b * 64, s);
                if (gm != 0x88888888u) {
#pragma unroll
                    for (int gi = 0; gi < 8; gi++) {
                        const uint32_t nv = (gm >> (4 * gi)) & 15u;
                        if (nv != 8u) {
#pragma unroll
                            for (int i = 0; i < 8; i++)
                                if ((uint32_t)i >= nv) s[8 * gi + i] = __float_as_uint(-INFINITY);
                        }
                    }
                }
                // row max: four independent chains of 3-input max (short dependences)
                float mq[4];
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    float m = fmaxf(__uint_as_float(s[16 * q]), __uint_as_float(s[16 * q + 1]));
#pragma unroll
                    for (int i = 2; i < 16; i += 2)
                        m = max3(m, __uint_as_float(s[16 * q + i]), __uint_as_float(s[16 * q + i + 1]));
                    mq[q] = m;
                }
                const float mx = fmaxf(max3(mq[0], mq[1], mq[2]), mq[3]);
                const float m_new = mx * sc;
                if (j == 0) m_ref = m_new;
                // Move the reference max (and rescale O_t) only when it grew by
                // more than 2^8; warp-uniform because TMEM access is collective.
                // PV_t(j-1) may still be accumulating into O_t: wait for it.  Its
                // pv_bar phase is unambiguous here: PV_t(j-2) is complete (S_t(j)
                // was issued after it) and PV_t(j) is not issued yet.
                if (j > 0 && __any_sync(0xffffffffu, m_new > m_ref + 8.f)) {
                    if (!wait_warp(pv_bar + t, (c - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const float m_to = fmaxf(m_ref, m_new);
                    const float f = ex2_approx(m_ref - m_to);
                    l0 *= f;
                    l1 *= f;
#pragma unroll
                    for (int pc = 0; pc < D / 32; pc++) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + pc * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                        tmem_st32(o_addr + pc * 32, o);
                    }
                    tmem_st_wait();
                    m_ref = m_to;
                }
                const float nm = -m_ref;
                uint32_t pk[32];
                // row sum in four partial sums (two packed pairs, short dependences),
                // folded into l0/l1.  All exponentials go to the MUFU pipe: the
                // softmax is issue-bound, and an FMA-pipe polynomial for part of
                // them cost more issue slots than it saved (measured on B200).
                float la[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    float x0, x1;
                    fma2(x0, x1, __uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]), sc, nm);
                    const float e0 = ex2_approx(x0);
                    const float e1 = ex2_approx(x1);
                    add2(la[2 * (i & 1)], la[2 * (i & 1) + 1], e0, e1);
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
                    pk[i] = *reinterpret_cast<uint32_t *>(&b2);
                }
                l0 += la[0] + la[2];
                l1 += la[1] + la[3];
                tmem_st32(s_base + b * 64, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(p_full + 2 * t + b);
            }
            if (!ok) break;
            // epilogue: O_t / l once the last P.V is done, rows scattered back to
            // token order.  (A parity wait on pv_bar cannot tell that phase from
            // the one before it while P.V(j-1) may still run, hence o_done.)
            if (!wait_warp(o_done + t, items_done & 1, abort_flag, p.status)) { ok = false; break; }
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
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn2)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static int bf16_map2(EncodeTiledFn2 enc, CUtensorMap *m, const void *base, int rows, int cols, int box_rows) {
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

static int kv_maps(EncodeTiledFn2 enc, KVMaps *m, const void *base, int rows, int cols) {
    return (bf16_map2(enc, &m->m64, base, rows, cols, 64) || bf16_map2(enc, &m->m32, base, rows, cols, 32) ||
            bf16_map2(enc, &m->m16, base, rows, cols, 16) || bf16_map2(enc, &m->m8, base, rows, cols, 8))
               ? -1
               : 0;
}

template <int D>
static int launch2(const void *qg, const void *kg, const void *vg, const A2Params &p, int max_items, int num_sms,
                   void *encode_fn, cudaStream_t st) {
    using C = A2Cfg<D>;
    EncodeTiledFn2 enc = (EncodeTiledFn2)encode_fn;
    CUtensorMap mq;
    KVMaps mk, mv;
    const int rows = p.H * p.N;
    if (bf16_map2(enc, &mq, qg, rows, D, 128) || kv_maps(enc, &mk, kg, rows, D) || kv_maps(enc, &mv, vg, rows, D))
        return -1;
    static int checked = 0;  // 1 = ok, -1 = refused
    if (checked == 0) {
        // the register split assumes the launch budget ptxas gave the kernel;
        // a larger split would make setmaxnreg.inc wait forever, so refuse
        cudaFuncAttributes fa;
        checked = (cudaFuncGetAttributes(&fa, attn2_kernel<D>) == cudaSuccess && fa.numRegs == C::REGS_LAUNCH) ? 1 : -1;
        if (checked == 1)
            cudaFuncSetAttribute(attn2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    }
    if (checked != 1) return -1;
    int grid = max_items < num_sms ? max_items : num_sms;
    if (grid < 1) grid = 1;
    attn2_kernel<D><<<grid, C::NTHREADS, C::SMEM, st>>>(mq, mk, mv, p);
    note_launch();
    return 0;
}

int k_attention2(int D, int H, int N, const void *qg, const void *kg, const void *vg, const int32_t *qperm,
                 int kk_cap, int kq_cap, const int2 *runs, const int2 *run_info, const uint32_t *masks,
                 int max_chunks, const AttnItem *items,
                 const int32_t *n_items, int max_items, void *out, float *lse, int *status, int num_sms,
                 void *encode_fn, cudaStream_t st) {
    A2Params p;
    p.H = H;
    p.N = N;
    p.qperm = qperm;
    p.kk_cap = kk_cap;
    p.kq_cap = kq_cap;
    p.runs = runs;
    p.run_info = run_info;
    p.masks = masks;
    p.max_chunks = max_chunks;
    p.items = items;
    p.n_items = n_items;
    p.out = reinterpret_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = status;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    if (D == 64) return launch2<64>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
    return launch2<128>(qg, kg, vg, p, max_items, num_sms, encode_fn, st);
}

}  // namespace ac
