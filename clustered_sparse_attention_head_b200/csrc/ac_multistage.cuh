// Algorithm 1 per-head state and launchers (see ac_multistage.cu).
#pragma once
#include "ac_common.cuh"

namespace ac {

struct MsHead {
    int nc;      // |C|: clusters created so far
    int nu;      // |U|: tokens still to be clustered
    int stage;   // t
    int flag;    // F
    int mt;      // m_t of the stage in progress
    int done;
    int same;    // the last stage removed no token (every later stage repeats it)
    int rep_src, rep_n;  // repeat to copy: centres [rep_src, rep_src + mt) rep_n more times
    int pad;
    double tau;
};

// N = row stride of a head; nrows = tokens clustered (the first nrows of each head)
void k_ms_init(int H, int N, int nrows, MsHead *st, int32_t *U, int32_t *U2, cudaStream_t s);
void k_ms_control(int H, int N, int m0, int nmax, int cap, MsHead *st, HeadSeg *seg, int32_t *info, int *status,
                  cudaStream_t s);
void k_ms_tau(int H, int N, int rule, double x, const HeadSeg *seg, const double *dist, const int32_t *perm,
              const int32_t *off, int cap, int kmax, MsHead *st, cudaStream_t s);
void k_ms_remove(int H, int N, const HeadSeg *seg, const double *dist, const int32_t *U, int32_t *Unext, MsHead *st,
                 cudaStream_t s);
// Copies the centres of a repeated stage (MsHead.rep_*) and clears the request.
void k_ms_repeat(int H, int D, MsHead *st, float *cent, int cap, cudaStream_t s);
// The distinct centres of each head's final set, in id order: cu [H, cap, D]
// (ku of them), cmap [H, cap] their ids, segu the pass descriptors over cu.
// Ties in the final reassignment go to the lowest id, which is always the first
// of identical centres, so assigning over cu and mapping back through cmap gives
// the assignment over the whole set.
void k_dedup_cent(int H, int D, const HeadSeg *seg, const float *cent, int cap, float *cu, int32_t *cmap,
                  HeadSeg *segu, cudaStream_t s);
void k_map_ids(int H, int N, const HeadSeg *seg, const int32_t *cmap, int cap, int32_t *assign, cudaStream_t s);
// Every remaining single-cluster stage of each head on chip (one CTA per
// head); wc: [H, wrows, D] doubles of scratch, wrows >= the largest |U| with
// m_t = 1 (N / m0).  A head whose |U| exceeds wrows is left to the host loop.
int k_ms_single(const void *x, int dtype, int H, int N, int D, int nrows, int m0, int nmax, int cap_c, int iters,
                const double *norm, int mode, int32_t *U, int32_t *U2, double *wc, int wrows, MsHead *st,
                float *cent, int cap, int *status, cudaStream_t s);
void k_ms_final(int H, int nrows, const MsHead *st, HeadSeg *seg, int32_t *ncl, uint8_t *flag, int32_t *info,
                cudaStream_t s);
void k_seg_uniform(int H, int nrows, int k, HeadSeg *seg, int32_t *ncl, uint8_t *flag, cudaStream_t s);
// Pass descriptors from per-head counts ncl (NULL: kfix for every head) less
// sub; counts outside [0, cap] are clamped and record ST_INVALID in status.
void k_seg_from_counts(int H, int nrows, const int32_t *ncl, int kfix, int cap, HeadSeg *seg, int *status,
                       cudaStream_t s, int sub = 0);
// The text-key group (ac_config.text_keys): rows [nrows, N) get id seg.k, count
// N - nrows, and ncl = seg.k + 1.
void k_text_group(int H, int N, int nrows, const HeadSeg *seg, int32_t *assign, int32_t *count, int cap,
                  int32_t *ncl, cudaStream_t s);

}  // namespace ac
