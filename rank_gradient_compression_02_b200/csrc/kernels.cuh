// The streaming kernels of one PowerSGD step (grouped over all layers).
//
//   pass A: M_w = G_w + E_w (stored over E_w), partial P = sum_w M_w Q per
//           (row, column chunk); the last CTA of a row block sums the chunk
//           partials into P_bar and a float64 Gram partial; the last row
//           block of a layer factors the Gram matrix (Cholesky QR) into T.
//   pass B: P_hat = P_bar T for the tile's rows; partial Q = sum_w M_w^T P_hat
//           per (row block, column); the last CTA of a column chunk sums the
//           row-block partials into Q_bar.
//   pass C: rec = P_hat Q_bar^T per element; E'_w = M_w - rec, optional
//           G_hat = rec, optional momentum.
//
// Step order from "anthology-of-the-sota" note-152 on PowerSGD, "Method".
// Every cross-CTA sum runs in a fixed order, so results are bitwise
// reproducible.  No CTA waits on another: the last CTA to arrive at a
// counter does the reduction.
#pragma once

#include "device_common.cuh"

namespace psgd {

// ---------------------------------------------------------------------------
// tile decode
struct TileCoord {
    int l, rb, c;
};

// The Q pass (REVERSE) walks the tiles backwards, the other passes
// forwards, so that each pass starts on the tiles the previous one touched
// last, whose lines are still in L2.  The direction is a template argument:
// a run-time select costs the first pass registers it does not have.
template <bool REVERSE>
__device__ __forceinline__ int tile_index() {
    if constexpr (REVERSE) return static_cast<int>(gridDim.x - 1 - blockIdx.x);
    else return static_cast<int>(blockIdx.x);
}

__device__ __forceinline__ TileCoord decode_tile(const LayerDesc& d, int t, int l) {
    const int local = static_cast<int>(t - d.tile_begin);
    TileCoord tc;
    tc.l = l;
    tc.rb = local / d.nchunk;
    tc.c = local - tc.rb * d.nchunk;
    return tc;
}

// ---------------------------------------------------------------------------
// orthogonalisation: factor the r x r Gram matrix (float64) with one warp.
// Cholesky G = R^T R column by column; column j is dropped (row j of R and
// column j of T set to zero) if its pivot, the squared norm of p_bar_j after
// projection on the kept columns before it, is <= drop_tol * max_k G_kk.
// T = R^-1 on the kept columns, so P_hat = P_bar T.
template <int R>
__device__ void factor_gram_warp(const double* Gs, double* Rs, double* Ts, int* drop, int r, double drop_tol,
                                 int lane) {
    for (int idx = lane; idx < R * R; idx += 32) {
        Rs[idx] = 0.0;
        Ts[idx] = 0.0;
    }
    __syncwarp();
    double maxd = 0.0;
    for (int k = 0; k < r; ++k) maxd = fmax(maxd, Gs[k * R + k]);
    const double tau = drop_tol * maxd;
    for (int j = 0; j < r; ++j) {
        double d = Gs[j * R + j];
        for (int k = 0; k < j; ++k) d -= Rs[k * R + j] * Rs[k * R + j];
        const bool dropped = (d <= tau);
        const double rjj = dropped ? 0.0 : sqrt(d);
        const int i = lane;
        if (i > j && i < r) {
            double s = Gs[j * R + i];
            for (int k = 0; k < j; ++k) s -= Rs[k * R + j] * Rs[k * R + i];
            Rs[j * R + i] = dropped ? 0.0 : s / rjj;
        }
        __syncwarp();
        if (lane == 0) {
            Rs[j * R + j] = rjj;
            drop[j] = dropped ? 1 : 0;
        }
        __syncwarp();
    }
    for (int j = 0; j < r; ++j) {
        const int l = lane;
        if (l <= j) {
            double t;
            if (drop[j]) {
                t = 0.0;
            } else if (l == j) {
                t = 1.0 / Rs[j * R + j];
            } else {
                double s = 0.0;
                for (int k = l; k < j; ++k) s += Ts[l * R + k] * Rs[k * R + j];
                t = -s / Rs[j * R + j];
            }
            Ts[l * R + j] = t;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// pass A

// Rank 32 uses the rank-lane kernels (one lane per rank index, M rows
// parked in shared memory and read as broadcasts); they walk a chunk (up to
// 32 * VEC columns) in sub-chunks of 32 columns.
template <int R>
struct IsWide { static constexpr bool value = R >= 32; };
constexpr int kWideCols = 32;
constexpr int kWideRows = 64;    // rows per tile cap for the rank-lane kernels

template <int R>
struct SmemA {
    // layout inside dynamic shared memory (bytes)
    static __host__ __device__ size_t ptr_bytes(int W) { return static_cast<size_t>(2 * W) * sizeof(void*); }
    static __host__ __device__ size_t rows_bytes(int tm) { return static_cast<size_t>(tm) * R * sizeof(double); }
    static __host__ __device__ size_t fac_bytes() { return 3 * R * R * sizeof(double) + 2 * R * sizeof(int) + 64; }
    // rank-lane kernel: every warp's parked rows (tm x 32 floats in all)
    static __host__ __device__ size_t wide_bytes(int tm) {
        (void)tm;
        return IsWide<R>::value ? static_cast<size_t>(kWideRows * kWideCols) * sizeof(float) : 0;
    }
    static __host__ __device__ size_t total(int W, int tm) {
        return ((ptr_bytes(W) + 15) & ~size_t(15)) + ((rows_bytes(tm) + 15) & ~size_t(15)) +
               ((fac_bytes() + 15) & ~size_t(15)) + wide_bytes(tm);
    }
};

template <int R, int VEC, typename GT, bool LAZY, bool SF, bool READM>
__device__ __forceinline__ void pass_a_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            const GT* const* gp, float* const* ep, const float* ph_prev) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = p.r;
    const int W = p.workers;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int64_t i1 = min(i0 + d.tm, m);
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    const bool active = lane < ns;
    const int64_t j = static_cast<int64_t>(s0 + (active ? lane : 0)) * VEC;

    // warm-start Q rows of this lane's columns, zero-padded to R
    float qv[VEC][R];
    {
        const float* Q = p.t.q[tc.l];
#pragma unroll
        for (int v = 0; v < VEC; ++v)
#pragma unroll
            for (int k = 0; k < R; ++k) qv[v][k] = (active && k < r) ? Q[(j + v) * r + k] : 0.f;
    }
    // previous Q_bar for rebuilding E' (lazy representation)
    float qp[LAZY ? VEC : 1][LAZY ? R : 1];
    if constexpr (LAZY) {
        const float* Qb = p.ws.qbar + d.qrow_off;
#pragma unroll
        for (int v = 0; v < VEC; ++v)
#pragma unroll
            for (int k = 0; k < R; ++k) qp[v][k] = (active && p.use_prev) ? Qb[(j + v) * R + k] : 0.f;
    }

    double* ppart = p.ws.ppart + d.ppart_off;
    constexpr int U = (VEC == 4) ? 4 : 8;
    // products are summed in float32 over runs of 8 terms (F workers x VEC
    // columns), then added to the float64 row accumulator
    constexpr int F = 8 / VEC;
    static_assert(U % F == 0, "flush interval must divide the unroll");
    constexpr int LG = Log2<R>::value;

    for (int64_t i = i0 + warp; i < i1; i += kWarps) {
        double acc[R];
#pragma unroll
        for (int k = 0; k < R; ++k) acc[k] = 0.0;
        if (active) {
            const int64_t base = i * n + j;
            float rec[VEC];
            if constexpr (LAZY) {
                float ph[R];
#pragma unroll
                for (int k = 0; k < R; ++k) ph[k] = ph_prev[(i - i0) * R + k];
#pragma unroll
                for (int v = 0; v < VEC; ++v) rec[v] = recon_dot<R>(ph, qp[v]);
            }
            float msum[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) msum[v] = 0.f;
            // G workers' loads in flight, then M, the store and the products;
            // float32 runs are flushed every F workers (<= 8 terms)
            auto group = [&](auto GC, int w0) {
                constexpr int G = decltype(GC)::value;
                [[maybe_unused]] float g[G][VEC];
                float e[G][VEC];
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    if constexpr (!READM) ld_grad<GT, VEC>(gp[w0 + u] + base, g[u]);
                    ld_f32<VEC>(ep[w0 + u] + base, e[u]);
                }
                if constexpr (!READM) {
#pragma unroll
                    for (int u = 0; u < G; ++u) {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            float ev = e[u][v];
                            if constexpr (LAZY) ev = ev - rec[v];
                            e[u][v] = g[u][v] + ev;
                        }
                        st_f32<VEC>(ep[w0 + u] + base, e[u]);
                    }
                }
                if constexpr (SF) {
#pragma unroll
                    for (int u = 0; u < G; ++u)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) msum[v] += e[u][v];
                } else {
                    float pw[R];
#pragma unroll
                    for (int k = 0; k < R; ++k) pw[k] = 0.f;
#pragma unroll
                    for (int u = 0; u < G; ++u) {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) axpy<R>(pw, e[u][v], qv[v]);
                        if ((u + 1) % F == 0 || u + 1 == G) {
#pragma unroll
                            for (int k = 0; k < R; ++k) {
                                acc[k] += static_cast<double>(pw[k]);
                                pw[k] = 0.f;
                            }
                        }
                    }
                }
            };
            int w = 0;
            for (; w + U <= W; w += U) group(std::integral_constant<int, U>{}, w);
            if constexpr (U > 4) {
                if (w + 4 <= W) {
                    group(std::integral_constant<int, 4>{}, w);
                    w += 4;
                }
            }
            if constexpr (U > 2) {
                if (w + 2 <= W) {
                    group(std::integral_constant<int, 2>{}, w);
                    w += 2;
                }
            }
            if (w < W) group(std::integral_constant<int, 1>{}, w);
            if constexpr (SF) {
                float pw[R];
#pragma unroll
                for (int k = 0; k < R; ++k) pw[k] = 0.f;
#pragma unroll
                for (int v = 0; v < VEC; ++v)
                    axpy<R>(pw, msum[v], qv[v]);
#pragma unroll
                for (int k = 0; k < R; ++k) acc[k] = static_cast<double>(pw[k]);
            }
        }
        TransposeReduce<double, R, 16>::run(acc, lane);
        if ((lane & ((32 >> LG) - 1)) == 0) {
            const int k = lane >> (5 - LG);
            ppart[(static_cast<int64_t>(tc.c) * m + i) * R + k] = acc[0];
        }
    }
}

// Rank-lane variant of the first pass (R = 32): lane k owns rank index k.
// Warp w owns rows w, w + 8, ... of the tile and stages them itself: for
// every (sub-chunk of 32 columns, worker) it forms M = G + E for its rows
// (a lane per column; M is stored over E), parks them in its own slice of
// shared memory, prefetches the next (sub-chunk, worker) into registers and
// then walks the parked rows, reading M as broadcasts against its slice of
// Q held in registers.  No CTA-wide barrier in the loop.  Products are
// summed in float32 over runs of 8 terms and flushed to a float64 per-row
// accumulator; the row's partial over the chunk needs no lane reduction.
template <int R, typename GT, bool LAZY, bool SF, bool READM>
__device__ __forceinline__ void pass_a_wide(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            const GT* const* gp, float* const* ep, const float* ph_prev,
                                            float* m_s) {
    static_assert(R == 32, "rank-lane kernels map one lane per rank index");
    constexpr int RPL = kWideRows / kWarps;   // rows per warp, at most
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = lane;
    const int r = p.r;
    const int W = p.workers;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * d.vec;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * d.vec, n - jc));
    const int nsc = (width + kWideCols - 1) / kWideCols;
    const int total = nsc * W;
    const float* Q = p.t.q[tc.l];
    const float* Qb = p.ws.qbar + d.qrow_off;
    float* ms_w = m_s + warp * RPL * kWideCols;

    float gv[RPL], ev[RPL];
    auto load = [&](int it) {
        const int sc = it / W, w = it - sc * W;
        const int64_t j0 = jc + sc * kWideCols;
        const int ncols = min(kWideCols, width - sc * kWideCols);
#pragma unroll
        for (int t = 0; t < RPL; ++t) {
            const int ii = warp + kWarps * t;
            gv[t] = 0.f;
            ev[t] = 0.f;
            if (ii < rows && lane < ncols) {
                const int64_t off = (i0 + ii) * n + j0 + lane;
                ev[t] = __ldcs(ep[w] + off);
                if constexpr (!READM) {
                    float g1[1];
                    ld_grad<GT, 1>(gp[w] + off, g1);
                    gv[t] = g1[0];
                }
            }
        }
    };

    double acc[RPL];
#pragma unroll
    for (int t = 0; t < RPL; ++t) acc[t] = 0.0;
    float qreg[kWideCols];
    float rec[LAZY ? RPL : 1];
    float msum[SF ? RPL : 1];

    // two float32 runs (even and odd columns) in one packed fp32x2 FMA, each
    // 8 terms long (16 columns), then both added to the float64 accumulator
    auto walk_rows = [&]() {
#pragma unroll
        for (int t = 0; t < RPL; ++t) {
            const int ii = warp + kWarps * t;
            if (ii < rows) {
                const float4* mrow = reinterpret_cast<const float4*>(ms_w + t * kWideCols);
                float2 run = make_float2(0.f, 0.f);
#pragma unroll
                for (int q4 = 0; q4 < kWideCols / 4; ++q4) {
                    const float4 mv = mrow[q4];
                    run = __ffma2_rn(make_float2(mv.x, mv.y), make_float2(qreg[4 * q4 + 0], qreg[4 * q4 + 1]), run);
                    run = __ffma2_rn(make_float2(mv.z, mv.w), make_float2(qreg[4 * q4 + 2], qreg[4 * q4 + 3]), run);
                    if ((q4 & 3) == 3) {
                        acc[t] += static_cast<double>(run.x) + static_cast<double>(run.y);
                        run = make_float2(0.f, 0.f);
                    }
                }
            }
        }
    };

    load(0);
    for (int it = 0; it < total; ++it) {
        const int sc = it / W, w = it - sc * W;
        const int64_t j0 = jc + sc * kWideCols;
        const int ncols = min(kWideCols, width - sc * kWideCols);
        if (w == 0) {
            // this lane's slice of Q for the sub-chunk: Q[j0 + jj][k]
#pragma unroll
            for (int jj = 0; jj < kWideCols; ++jj) qreg[jj] = (jj < ncols && k < r) ? Q[(j0 + jj) * r + k] : 0.f;
            if constexpr (LAZY) {
                // the previous step's reconstruction of (row, this lane's column)
                float qp[R];
#pragma unroll
                for (int kk = 0; kk < R; ++kk)
                    qp[kk] = (lane < ncols && p.use_prev) ? Qb[(j0 + lane) * R + kk] : 0.f;
#pragma unroll
                for (int t = 0; t < RPL; ++t) {
                    // recon_dot's operation order, P_hat row read from shared memory
                    const int ii = min(warp + kWarps * t, rows - 1);
                    float s2 = 0.f;
#pragma unroll
                    for (int kk = 0; kk < R; ++kk) s2 = fmaf(ph_prev[ii * R + kk], qp[kk], s2);
                    rec[t] = s2;
                }
            }
            if constexpr (SF) {
#pragma unroll
                for (int t = 0; t < RPL; ++t) msum[t] = 0.f;
            }
        }
        // M for this worker's rows
#pragma unroll
        for (int t = 0; t < RPL; ++t) {
            const int ii = warp + kWarps * t;
            float mval = ev[t];
            if (ii < rows && lane < ncols) {
                if constexpr (!READM) {
                    float e2 = ev[t];
                    if constexpr (LAZY) e2 = e2 - rec[t];
                    mval = gv[t] + e2;
                    ep[w][(i0 + ii) * n + j0 + lane] = mval;
                }
            } else {
                mval = 0.f;
            }
            if constexpr (SF) {
                msum[t] += mval;
            } else {
                ms_w[t * kWideCols + lane] = mval;
            }
        }
        if (it + 1 < total) load(it + 1);   // in flight while the rows are walked
        if constexpr (SF) {
            if (w == W - 1) {
#pragma unroll
                for (int t = 0; t < RPL; ++t) ms_w[t * kWideCols + lane] = msum[t];
                __syncwarp();
                walk_rows();
                __syncwarp();
            }
        } else {
            __syncwarp();
            walk_rows();
            __syncwarp();
        }
    }
    double* ppart = p.ws.ppart + d.ppart_off;
#pragma unroll
    for (int t = 0; t < RPL; ++t) {
        const int ii = warp + kWarps * t;
        if (ii < rows) ppart[(static_cast<int64_t>(tc.c) * m + i0 + ii) * R + k] = acc[t];
    }
}

// Last CTA of a row block: P_bar rows and the Gram partial.  Last row block
// of a layer: Gram sum and factorisation.
template <int R>
__device__ void pass_a_epilogue(const Params& p, const LayerDesc& d, const TileCoord& tc, double* pb_s,
                                unsigned char* fac) {
    __shared__ int s_flag;
    constexpr int NG = R * (R + 1) / 2;
    const int tid = threadIdx.x;
    const CounterLayout cl = counter_layout(d.nrb, d.nsup, d.nchunk);
    unsigned* cnt = p.ws.cnt + d.cnt_off;

    // 1) the last chunk tile of a row block: P_bar rows and the Gram partial
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.a_rb + tc.rb], 1u);
        if (prev >= static_cast<unsigned>(d.nchunk)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(d.nchunk - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();

    const int64_t m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), m - i0));
    const double* ppart = p.ws.ppart + d.ppart_off;
    double* pbar = p.ws.pbar + d.prow_off;
    const double inv_w = 1.0 / static_cast<double>(p.workers);
    for (int idx = tid; idx < rows * R; idx += kThreads) {
        const int64_t i = i0 + idx / R;
        const int k = idx % R;
        double s = 0.0;
        for (int c = 0; c < d.nchunk; ++c) s += __ldcg(&ppart[(static_cast<int64_t>(c) * m + i) * R + k]);
        if (p.dist) {
            // this rank's share of the all-reduce: the row's sum over its workers
            p.dist_out[d.prow_off + i * R + k] = s;
            continue;
        }
        const double v = s * inv_w;
        pb_s[idx] = v;
        pbar[i * R + k] = v;
    }
    if (tid == 0) cnt[cl.a_rb + tc.rb] = 0u;
    if (p.dist) return;
    __syncthreads();

    double* gram = p.ws.gram + d.gram_off;
    for (int pidx = tid; pidx < NG; pidx += kThreads) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = 0.0;
        for (int ii = 0; ii < rows; ++ii) s += pb_s[ii * R + a] * pb_s[ii * R + b];
        gram[static_cast<int64_t>(tc.rb) * NG + pidx] = s;
    }

    // 2) the last row block of a super-block: sum its Gram partials
    const int sup = tc.rb / kSuper;
    const int rb0 = sup * kSuper;
    const int nin = min(kSuper, d.nrb - rb0);
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.a_sup + sup], 1u);
        if (prev >= static_cast<unsigned>(nin)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(nin - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    double* gsup = p.ws.gsup + d.gsup_off;
    for (int pidx = tid; pidx < NG; pidx += kThreads) {
        double s = 0.0;
        for (int k = 0; k < nin; ++k) s += __ldcg(&gram[static_cast<int64_t>(rb0 + k) * NG + pidx]);
        gsup[static_cast<int64_t>(sup) * NG + pidx] = s;
    }
    if (tid == 0) cnt[cl.a_sup + sup] = 0u;

    // 3) the last super-block of the layer: Gram sum and factorisation
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.a_layer], 1u);
        if (prev >= static_cast<unsigned>(d.nsup)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(d.nsup - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();

    double* Gs = reinterpret_cast<double*>(fac);
    double* Rs = Gs + R * R;
    double* Ts = Rs + R * R;
    int* drop = reinterpret_cast<int*>(Ts + R * R);
    for (int pidx = tid; pidx < NG; pidx += kThreads) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = 0.0;
        for (int k = 0; k < d.nsup; ++k) s += __ldcg(&gsup[static_cast<int64_t>(k) * NG + pidx]);
        Gs[a * R + b] = s;
        Gs[b * R + a] = s;
    }
    __syncthreads();
    if (tid < 32) {
        factor_gram_warp<R>(Gs, Rs, Ts, drop, p.r, p.drop_tol, tid);
        double* T = p.ws.T + d.t_off;
        for (int idx = tid; idx < R * R; idx += 32) T[idx] = Ts[idx];
    }
    if (tid == 0) cnt[cl.a_layer] = 0u;
}

// READM: a later power iteration of the same step; M is already in the
// error buffers, so only M is read (no gradient, no store).
template <int R, typename GT, bool LAZY, bool SF, bool READM>
__global__ void __launch_bounds__(kThreads, (R <= 8 ? 3 : 2)) k_pass_a(Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int t = tile_index<false>();
    const int l = p.t.tile_layer[t];
    const LayerDesc d = p.t.layers[l];
    const TileCoord tc = decode_tile(d, t, l);
    const int W = p.workers;
    const int L = p.num_layers;

    const GT** gp = reinterpret_cast<const GT**>(smem);
    float** ep = reinterpret_cast<float**>(smem + static_cast<size_t>(W) * sizeof(void*));
    double* rows_d = reinterpret_cast<double*>(smem + ((SmemA<R>::ptr_bytes(W) + 15) & ~size_t(15)));
    float* rows_s = reinterpret_cast<float*>(rows_d);
    unsigned char* fac = reinterpret_cast<unsigned char*>(rows_d) + ((SmemA<R>::rows_bytes(d.tm) + 15) & ~size_t(15));
    float* wide = reinterpret_cast<float*>(fac + ((SmemA<R>::fac_bytes() + 15) & ~size_t(15)));

    for (int w = threadIdx.x; w < W; w += kThreads) {
        gp[w] = static_cast<const GT*>(p.t.grads[w * L + l]);
        ep[w] = p.t.errors[w * L + l];
    }
    if constexpr (LAZY) {
        const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
        const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
        const float* ph = p.ws.phat + d.prow_off + i0 * R;
        for (int idx = threadIdx.x; idx < rows * R; idx += kThreads) rows_s[idx] = p.use_prev ? ph[idx] : 0.f;
    }
    __syncthreads();

    if constexpr (IsWide<R>::value) {
        pass_a_wide<R, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s, wide);
    } else {
        // VEC x R values of Q live in registers: VEC = 4 up to R = 4, 2 up to 16
        if (d.vec == 4) {
            if constexpr (R <= 4) pass_a_rows<R, 4, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s);
        } else if (d.vec == 2) {
            if constexpr (R <= 16) pass_a_rows<R, 2, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s);
        } else {
            pass_a_rows<R, 1, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s);
        }
    }
    pass_a_epilogue<R>(p, d, tc, rows_d, fac);
}

// ---------------------------------------------------------------------------
// pass B

template <int R>
struct SmemB {
    static __host__ __device__ size_t ptr_bytes(int W) { return static_cast<size_t>(W) * sizeof(void*); }
    static __host__ __device__ size_t rows_bytes(int tm) { return static_cast<size_t>(tm) * R * sizeof(float); }
    static __host__ __device__ size_t t_bytes() { return R * R * sizeof(double); }
    static __host__ __device__ size_t red_bytes(int vec) {
        if (IsWide<R>::value) {
            // rank-lane kernel: parked rows (tm x 32) + warp partials (8 x 32 x R)
            return static_cast<size_t>(kWideRows * kWideCols + kWarps * kWideCols * R) * sizeof(float);
        }
        return static_cast<size_t>(kWarps) * R * vec * 32 * sizeof(float);
    }
    static __host__ __device__ size_t total(int W, int tm, int vec) {
        return ((ptr_bytes(W) + 15) & ~size_t(15)) + ((rows_bytes(tm) + 15) & ~size_t(15)) + t_bytes() +
               red_bytes(vec);
    }
};

// P_hat rows [i0, i0+rows) of a layer into shared memory: P_bar T, float64
// accumulation in column order.  Chunk 0 also writes them out.
template <int R>
__device__ __forceinline__ void load_phat_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                               float* ph_s, double* T_s, bool write_out) {
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
    const double* T = p.ws.T + d.t_off;
    for (int idx = threadIdx.x; idx < R * R; idx += kThreads) T_s[idx] = T[idx];
    __syncthreads();
    const double* pbar = p.ws.pbar + d.prow_off + i0 * R;
    float* phat_ws = p.ws.phat + d.prow_off + i0 * R;
    float* out = (p.t.p_hat_out != nullptr) ? p.t.p_hat_out[tc.l] : nullptr;
    const int r = p.r;
    for (int idx = threadIdx.x; idx < rows * R; idx += kThreads) {
        const int ii = idx / R;
        const int k = idx % R;
        double s = 0.0;
        for (int a = 0; a <= k; ++a) s += pbar[ii * R + a] * T_s[a * R + k];
        const float v = static_cast<float>(s);
        ph_s[idx] = v;
        if (write_out) {
            phat_ws[idx] = v;
            if (out != nullptr && k < r) out[(i0 + ii) * r + k] = v;
        }
    }
    __syncthreads();
}

template <int R, int VEC, bool SF>
__device__ __forceinline__ void pass_b_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            float* const* ep, const float* ph_s, float* red_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int W = p.workers;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int64_t i1 = min(i0 + d.tm, m);
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    const bool active = lane < ns;
    const int64_t j = static_cast<int64_t>(s0 + (active ? lane : 0)) * VEC;
    constexpr int U = 8;   // 8 workers' loads in flight per lane (pass B only reads)

    float qacc[VEC][R];
#pragma unroll
    for (int v = 0; v < VEC; ++v)
#pragma unroll
        for (int k = 0; k < R; ++k) qacc[v][k] = 0.f;

    if (active) {
        for (int64_t i = i0 + warp; i < i1; i += kWarps) {
            float ph[R];
#pragma unroll
            for (int k = 0; k < R; ++k) ph[k] = ph_s[(i - i0) * R + k];
            const int64_t base = i * n + j;
            float msum[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) msum[v] = 0.f;
            // G workers' loads in flight, then their products
            auto group = [&](auto GC, int w0) {
                constexpr int G = decltype(GC)::value;
                float e[G][VEC];
#pragma unroll
                for (int u = 0; u < G; ++u) ld_f32<VEC>(ep[w0 + u] + base, e[u]);
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    if constexpr (SF) {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) msum[v] += e[u][v];
                    } else {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) axpy<R>(qacc[v], e[u][v], ph);
                    }
                }
            };
            int w = 0;
            for (; w + U <= W; w += U) group(std::integral_constant<int, U>{}, w);
            if (w + 4 <= W) {
                group(std::integral_constant<int, 4>{}, w);
                w += 4;
            }
            if (w + 2 <= W) {
                group(std::integral_constant<int, 2>{}, w);
                w += 2;
            }
            if (w < W) group(std::integral_constant<int, 1>{}, w);
            if constexpr (SF) {
#pragma unroll
                for (int v = 0; v < VEC; ++v)
                    axpy<R>(qacc[v], msum[v], ph);
            }
        }
    }
    // this warp's partial, laid out [warp][k][v][lane] (conflict-free)
#pragma unroll
    for (int k = 0; k < R; ++k)
#pragma unroll
        for (int v = 0; v < VEC; ++v) red_s[((warp * R + k) * VEC + v) * 32 + lane] = qacc[v][k];
    __syncthreads();
    // sum over warps in order; write the row block's partial Q rows
    double* qpart = p.ws.qpart + d.qpart_off;
    const int cols = ns * VEC;
    for (int idx = threadIdx.x; idx < cols * R; idx += kThreads) {
        const int cc = idx / R;        // local column
        const int k = idx % R;
        const int ln = cc / VEC, v = cc % VEC;
        double s = 0.0;
#pragma unroll
        for (int wp = 0; wp < kWarps; ++wp) s += static_cast<double>(red_s[((wp * R + k) * VEC + v) * 32 + ln]);
        qpart[(static_cast<int64_t>(tc.rb) * n + static_cast<int64_t>(s0) * VEC + cc) * R + k] = s;
    }
}

// Rank-lane variant of the second pass (R = 32): lane k owns rank index k
// and warp w rows w, w + 8, ... of the tile.  For every sub-chunk of 32
// columns and every worker a warp parks its M rows in its own slice of
// shared memory (prefetching the next ones into registers) and accumulates,
// in float32, M[i][c] * P_hat[i][k] for its 32 columns; at the end of a
// sub-chunk the 8 warps' partials are summed in float64 in warp order.
template <int R, bool SF>
__device__ __forceinline__ void pass_b_wide(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            float* const* ep, const float* ph_s, float* sm) {
    static_assert(R == 32, "rank-lane kernels map one lane per rank index");
    constexpr int RPL = kWideRows / kWarps;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = lane;
    const int W = p.workers;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * d.vec;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * d.vec, n - jc));
    const int nsc = (width + kWideCols - 1) / kWideCols;
    float* ms_w = sm + warp * RPL * kWideCols;               // parked rows
    float* red_s = sm + kWideRows * kWideCols;               // [warp][column][k]
    double* qpart = p.ws.qpart + d.qpart_off;

    float ph[RPL];
#pragma unroll
    for (int t = 0; t < RPL; ++t) {
        const int ii = warp + kWarps * t;
        ph[t] = (ii < rows) ? ph_s[ii * R + k] : 0.f;
    }
    float mv_in[RPL];
    auto load = [&](int it) {
        const int sc = it / W, w = it - sc * W;
        const int ncols = min(kWideCols, width - sc * kWideCols);
#pragma unroll
        for (int t = 0; t < RPL; ++t) {
            const int ii = warp + kWarps * t;
            mv_in[t] = (ii < rows && lane < ncols) ? __ldcs(ep[w] + (i0 + ii) * n + jc + sc * kWideCols + lane) : 0.f;
        }
    };
    const int total = nsc * W;
    load(0);
    float2 acc[kWideCols / 2];   // columns (2c, 2c + 1)
    float msum[SF ? RPL : 1];
    for (int it = 0; it < total; ++it) {
        const int sc = it / W, w = it - sc * W;
        if (w == 0) {
#pragma unroll
            for (int c = 0; c < kWideCols / 2; ++c) acc[c] = make_float2(0.f, 0.f);
            if constexpr (SF) {
#pragma unroll
                for (int t = 0; t < RPL; ++t) msum[t] = 0.f;
            }
        }
        bool walk = true;
        if constexpr (SF) {
#pragma unroll
            for (int t = 0; t < RPL; ++t) msum[t] += mv_in[t];
            walk = (w == W - 1);
            if (walk) {
#pragma unroll
                for (int t = 0; t < RPL; ++t) ms_w[t * kWideCols + lane] = msum[t];
            }
        } else {
#pragma unroll
            for (int t = 0; t < RPL; ++t) ms_w[t * kWideCols + lane] = mv_in[t];
        }
        if (it + 1 < total) load(it + 1);
        if (walk) {
            __syncwarp();
#pragma unroll
            for (int t = 0; t < RPL; ++t) {
                const float4* mrow = reinterpret_cast<const float4*>(ms_w + t * kWideCols);
                const float2 pp = make_float2(ph[t], ph[t]);
#pragma unroll
                for (int c4 = 0; c4 < kWideCols / 4; ++c4) {
                    const float4 mv = mrow[c4];
                    acc[2 * c4 + 0] = __ffma2_rn(make_float2(mv.x, mv.y), pp, acc[2 * c4 + 0]);
                    acc[2 * c4 + 1] = __ffma2_rn(make_float2(mv.z, mv.w), pp, acc[2 * c4 + 1]);
                }
            }
            __syncwarp();
        }
        if (w == W - 1) {
            // sub-chunk done: sum the warps' partials in warp order
#pragma unroll
            for (int c = 0; c < kWideCols / 2; ++c) {
                red_s[(warp * kWideCols + 2 * c) * R + k] = acc[c].x;
                red_s[(warp * kWideCols + 2 * c + 1) * R + k] = acc[c].y;
            }
            __syncthreads();
            const int ncols = min(kWideCols, width - sc * kWideCols);
            for (int idx = tid; idx < ncols * R; idx += kThreads) {
                const int c = idx / R, kk = idx % R;
                double s2 = 0.0;
#pragma unroll
                for (int wp = 0; wp < kWarps; ++wp) s2 += static_cast<double>(red_s[(wp * kWideCols + c) * R + kk]);
                qpart[(static_cast<int64_t>(tc.rb) * n + jc + sc * kWideCols + c) * R + kk] = s2;
            }
            __syncthreads();
        }
    }
}

template <int R>
__device__ void pass_b_epilogue(const Params& p, const LayerDesc& d, const TileCoord& tc) {
    __shared__ int s_flag;
    const int tid = threadIdx.x;
    const CounterLayout cl = counter_layout(d.nrb, d.nsup, d.nchunk);
    unsigned* cnt = p.ws.cnt + d.cnt_off;
    const int64_t n = d.n;
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    const int64_t col0 = static_cast<int64_t>(s0) * d.vec;
    const int cols = ns * d.vec;

    // 1) the last row block of a super-block (for this chunk): sum its partials
    const int sup = tc.rb / kSuper;
    const int rb0 = sup * kSuper;
    const int nin = min(kSuper, d.nrb - rb0);
    unsigned* c1 = &cnt[cl.b_sup + static_cast<int64_t>(tc.c) * d.nsup + sup];
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(c1, 1u);
        if (prev >= static_cast<unsigned>(nin)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(nin - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    const double* qpart = p.ws.qpart + d.qpart_off;
    double* qsup = p.ws.qsup + d.qsup_off;
    for (int idx = tid; idx < cols * R; idx += kThreads) {
        const int64_t col = col0 + idx / R;
        const int k = idx % R;
        double s = 0.0;
        for (int j = 0; j < nin; ++j) s += __ldcg(&qpart[(static_cast<int64_t>(rb0 + j) * n + col) * R + k]);
        qsup[(static_cast<int64_t>(sup) * n + col) * R + k] = s;
    }
    if (tid == 0) *c1 = 0u;

    // 2) the last super-block of the chunk: Q_bar for the chunk's columns
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.b_chunk + tc.c], 1u);
        if (prev >= static_cast<unsigned>(d.nsup)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(d.nsup - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    float* qbar = p.ws.qbar + d.qrow_off;
    float* qout = p.t.q[tc.l];
    const int r = p.r;
    const double inv_w = 1.0 / static_cast<double>(p.workers);
    for (int idx = tid; idx < cols * R; idx += kThreads) {
        const int64_t col = col0 + idx / R;
        const int k = idx % R;
        double s = 0.0;
        for (int j = 0; j < d.nsup; ++j) s += __ldcg(&qsup[(static_cast<int64_t>(j) * n + col) * R + k]);
        if (p.dist) {
            p.dist_out[d.qrow_off + col * R + k] = s;   // this rank's share of the all-reduce
            continue;
        }
        const float v = static_cast<float>(s * inv_w);
        qbar[col * R + k] = v;
        if (k < r) qout[col * r + k] = v;
    }
    if (tid == 0) cnt[cl.b_chunk + tc.c] = 0u;
}

template <int R, bool SF>
__global__ void __launch_bounds__(kThreads, (R <= 8 ? 3 : 2)) k_pass_b(Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int t = tile_index<true>();
    const int l = p.t.tile_layer[t];
    const LayerDesc d = p.t.layers[l];
    const TileCoord tc = decode_tile(d, t, l);
    const int W = p.workers;
    const int L = p.num_layers;

    float** ep = reinterpret_cast<float**>(smem);
    float* ph_s = reinterpret_cast<float*>(smem + ((SmemB<R>::ptr_bytes(W) + 15) & ~size_t(15)));
    double* T_s = reinterpret_cast<double*>(reinterpret_cast<unsigned char*>(ph_s) +
                                            ((SmemB<R>::rows_bytes(d.tm) + 15) & ~size_t(15)));
    float* red_s = reinterpret_cast<float*>(T_s + R * R);

    for (int w = threadIdx.x; w < W; w += kThreads) ep[w] = p.t.errors[w * L + l];
    load_phat_rows<R>(p, d, tc, ph_s, T_s, tc.c == 0);

    if constexpr (IsWide<R>::value) {
        pass_b_wide<R, SF>(p, d, tc, ep, ph_s, red_s);
    } else {
        if (d.vec == 4) {
            if constexpr (R <= 4) pass_b_rows<R, 4, SF>(p, d, tc, ep, ph_s, red_s);
        } else if (d.vec == 2) {
            if constexpr (R <= 16) pass_b_rows<R, 2, SF>(p, d, tc, ep, ph_s, red_s);
        } else {
            pass_b_rows<R, 1, SF>(p, d, tc, ep, ph_s, red_s);
        }
    }
    pass_b_epilogue<R>(p, d, tc);
}

// ---------------------------------------------------------------------------
// pass C: residual / decompression / momentum

template <int R>
struct SmemC {
    static __host__ __device__ size_t ptr_bytes(int W) { return static_cast<size_t>(W < 1 ? 1 : W) * sizeof(void*); }
    static __host__ __device__ size_t rows_bytes(int tm) { return static_cast<size_t>(tm) * R * sizeof(float); }
    static __host__ __device__ size_t wide_bytes() {
        return IsWide<R>::value ? static_cast<size_t>(R) * 4 * kWideCols * sizeof(float) : 0;
    }
    static __host__ __device__ size_t total(int W, int tm) {
        return ((ptr_bytes(W) + 15) & ~size_t(15)) + ((rows_bytes(tm) + 15) & ~size_t(15)) + wide_bytes();
    }
};

// Rank-lane variant of the third pass (R = 16 or 32).  The tile's
// reconstruction rec = P_hat Q_bar^T (rows x chunk width) is formed once
// from shared memory (Q_bar transposed, float4 per lane) with the same
// float32 operation order as recon_dot, then applied to every worker:
// thread (warp w, lane q) owns rows w + 8 s and columns 4q .. 4q+3.
template <int R>
__device__ __forceinline__ void pass_c_wide(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            float* const* ep, const float* ph_s, float* qt_s) {
    constexpr int STR = 4 * kWideCols;
    constexpr int SR = kWideRows / kWarps;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = p.do_resid ? p.workers : 0;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * d.vec;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * d.vec, n - jc));
    const float* Qb = p.ws.qbar + d.qrow_off;
    for (int idx = tid; idx < R * STR; idx += kThreads) {
        const int kk = idx / STR, jj = idx % STR;
        qt_s[idx] = (jj < width) ? Qb[(jc + jj) * R + kk] : 0.f;
    }
    __syncthreads();
    // rec[s][v] = sum_k ph[row_s][k] * qbar[col_v][k], k ascending (recon_dot's
    // order); four k at a time: Q_bar for them in registers, P_hat rows as
    // float4 broadcasts, two columns per packed FMA
    float2 rec2[SR][2];
#pragma unroll
    for (int s2 = 0; s2 < SR; ++s2) rec2[s2][0] = rec2[s2][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k4 = 0; k4 < R; k4 += 4) {
        float4 q[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) q[kk] = *reinterpret_cast<const float4*>(qt_s + (k4 + kk) * STR + 4 * lane);
#pragma unroll
        for (int s2 = 0; s2 < SR; ++s2) {
            const int ii = min(warp + kWarps * s2, rows - 1);
            const float4 ph = *reinterpret_cast<const float4*>(ph_s + ii * R + k4);
            const float phk[4] = {ph.x, ph.y, ph.z, ph.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float2 pp = make_float2(phk[kk], phk[kk]);
                rec2[s2][0] = __ffma2_rn(pp, make_float2(q[kk].x, q[kk].y), rec2[s2][0]);
                rec2[s2][1] = __ffma2_rn(pp, make_float2(q[kk].z, q[kk].w), rec2[s2][1]);
            }
        }
    }
    float rec[SR][4];
#pragma unroll
    for (int s2 = 0; s2 < SR; ++s2) {
        rec[s2][0] = rec2[s2][0].x;
        rec[s2][1] = rec2[s2][0].y;
        rec[s2][2] = rec2[s2][1].x;
        rec[s2][3] = rec2[s2][1].y;
    }
    float* recon = (p.do_recon && p.t.recon_out != nullptr) ? p.t.recon_out[tc.l] : nullptr;
    float* xs = p.do_mom ? p.t.params[tc.l] : nullptr;
    float* ms = p.do_mom ? p.t.mom[tc.l] : nullptr;
    const int jq = 4 * lane;
    if (jq >= width) return;
    const bool full4 = (d.vec == 4);   // 4 columns, 16-byte aligned
    const int nv = min(4, width - jq);
#pragma unroll
    for (int s2 = 0; s2 < SR; ++s2) {
        const int ii = warp + kWarps * s2;
        if (ii >= rows) break;
        const int64_t base = (i0 + ii) * n + jc + jq;
        auto apply = [&](float* ptr, auto&& op) {
            if (full4) {
                float4 v = *reinterpret_cast<float4*>(ptr + base);
                op(v.x, 0); op(v.y, 1); op(v.z, 2); op(v.w, 3);
                *reinterpret_cast<float4*>(ptr + base) = v;
            } else {
                for (int v = 0; v < nv; ++v) op(ptr[base + v], v);
            }
        };
        if (recon != nullptr) apply(recon, [&](float& x, int v) { x = rec[s2][v]; });
        if (xs != nullptr) {
            if (full4) {
                float4 mo = *reinterpret_cast<float4*>(ms + base);
                float4 x = *reinterpret_cast<float4*>(xs + base);
                mo.x = fmaf(p.beta, mo.x, rec[s2][0]); x.x = fmaf(-p.lr, mo.x, x.x);
                mo.y = fmaf(p.beta, mo.y, rec[s2][1]); x.y = fmaf(-p.lr, mo.y, x.y);
                mo.z = fmaf(p.beta, mo.z, rec[s2][2]); x.z = fmaf(-p.lr, mo.z, x.z);
                mo.w = fmaf(p.beta, mo.w, rec[s2][3]); x.w = fmaf(-p.lr, mo.w, x.w);
                *reinterpret_cast<float4*>(ms + base) = mo;
                *reinterpret_cast<float4*>(xs + base) = x;
            } else {
                for (int v = 0; v < nv; ++v) {
                    const float mo = fmaf(p.beta, ms[base + v], rec[s2][v]);
                    ms[base + v] = mo;
                    xs[base + v] = fmaf(-p.lr, mo, xs[base + v]);
                }
            }
        }
        for (int w = 0; w < W; ++w) apply(ep[w], [&](float& x, int v) { x = x - rec[s2][v]; });
    }
}

template <int R, int VEC>
__device__ __forceinline__ void pass_c_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            float* const* ep, const float* ph_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int W = p.do_resid ? p.workers : 0;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int64_t i1 = min(i0 + d.tm, m);
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    if (lane >= ns) return;
    const int64_t j = static_cast<int64_t>(s0 + lane) * VEC;
    constexpr int U = (VEC == 4) ? 4 : 8;

    float qb[VEC][R];
    {
        const float* Qb = p.ws.qbar + d.qrow_off;
#pragma unroll
        for (int v = 0; v < VEC; ++v)
#pragma unroll
            for (int k = 0; k < R; ++k) qb[v][k] = Qb[(j + v) * R + k];
    }
    float* recon = (p.do_recon && p.t.recon_out != nullptr) ? p.t.recon_out[tc.l] : nullptr;
    float* xs = p.do_mom ? p.t.params[tc.l] : nullptr;
    float* ms = p.do_mom ? p.t.mom[tc.l] : nullptr;

    for (int64_t i = i0 + warp; i < i1; i += kWarps) {
        float ph[R];
#pragma unroll
        for (int k = 0; k < R; ++k) ph[k] = ph_s[(i - i0) * R + k];
        float rec[VEC];
#pragma unroll
        for (int v = 0; v + 1 < VEC; v += 2) {
            const float2 r2 = recon_dot2<R>(ph, qb[v], qb[v + 1]);
            rec[v] = r2.x;
            rec[v + 1] = r2.y;
        }
        if constexpr (VEC == 1) rec[0] = recon_dot<R>(ph, qb[0]);
        const int64_t base = i * n + j;
        if (recon != nullptr) st_f32<VEC>(recon + base, rec);
        if (xs != nullptr) {
            float x[VEC], mo[VEC];
            ld_f32<VEC>(xs + base, x);
            ld_f32<VEC>(ms + base, mo);
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                mo[v] = fmaf(p.beta, mo[v], rec[v]);
                x[v] = fmaf(-p.lr, mo[v], x[v]);
            }
            st_f32<VEC>(ms + base, mo);
            st_f32<VEC>(xs + base, x);
        }
        auto group = [&](auto GC, int w0) {
            constexpr int G = decltype(GC)::value;
            float e[G][VEC];
#pragma unroll
            for (int u = 0; u < G; ++u) ld_f32<VEC>(ep[w0 + u] + base, e[u]);
#pragma unroll
            for (int u = 0; u < G; ++u) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) e[u][v] = e[u][v] - rec[v];
                st_f32<VEC>(ep[w0 + u] + base, e[u]);
            }
        };
        int w = 0;
        for (; w + U <= W; w += U) group(std::integral_constant<int, U>{}, w);
        if constexpr (U > 4) {
            if (w + 4 <= W) {
                group(std::integral_constant<int, 4>{}, w);
                w += 4;
            }
        }
        if (w + 2 <= W) {
            group(std::integral_constant<int, 2>{}, w);
            w += 2;
        }
        if (w < W) group(std::integral_constant<int, 1>{}, w);
    }
}

template <int R>
__global__ void __launch_bounds__(kThreads, 2) k_pass_c(Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int t = tile_index<false>();
    const int l = p.t.tile_layer[t];
    const LayerDesc d = p.t.layers[l];
    const TileCoord tc = decode_tile(d, t, l);
    const int W = p.workers;
    const int L = p.num_layers;
    float** ep = reinterpret_cast<float**>(smem);
    float* ph_s = reinterpret_cast<float*>(smem + ((SmemC<R>::ptr_bytes(W) + 15) & ~size_t(15)));
    float* qt_s = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(ph_s) +
                                           ((SmemC<R>::rows_bytes(d.tm) + 15) & ~size_t(15)));
    if (p.do_resid)
        for (int w = threadIdx.x; w < W; w += kThreads) ep[w] = p.t.errors[w * L + l];
    {
        const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
        const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
        const float* ph = p.ws.phat + d.prow_off + i0 * R;
        for (int idx = threadIdx.x; idx < rows * R; idx += kThreads) ph_s[idx] = ph[idx];
    }
    __syncthreads();
    if constexpr (IsWide<R>::value) {
        pass_c_wide<R>(p, d, tc, ep, ph_s, qt_s);
    } else {
        if (d.vec == 4) {
            if constexpr (R <= 4) pass_c_rows<R, 4>(p, d, tc, ep, ph_s);
        } else if (d.vec == 2) {
            if constexpr (R <= 16) pass_c_rows<R, 2>(p, d, tc, ep, ph_s);
        } else {
            pass_c_rows<R, 1>(p, d, tc, ep, ph_s);
        }
    }
}

// ---------------------------------------------------------------------------
// Distributed step, after the all-reduce of P: P_bar = (sum over all ranks'
// workers) / W_global, its Gram matrix (float64, pairs over warps, rows over
// lanes, fixed order) and the Cholesky factorisation into T.  One CTA per
// layer.
template <int R>
__global__ void __launch_bounds__(kThreads) k_dist_orth(Params p) {
    __shared__ double Gs[R * R];
    __shared__ double Rs[R * R];
    __shared__ double Ts[R * R];
    __shared__ int drop[R];
    const int l = blockIdx.x;
    const LayerDesc d = p.t.layers[l];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NG = R * (R + 1) / 2;
    double* pbar = p.ws.pbar + d.prow_off;
    const double* psum = p.dist_in + d.prow_off;
    for (int64_t idx = tid; idx < d.m * R; idx += kThreads) pbar[idx] = psum[idx] * p.inv_w_global;
    __syncthreads();
    for (int pidx = warp; pidx < NG; pidx += kWarps) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = 0.0;
        for (int64_t i = lane; i < d.m; i += 32) s += pbar[i * R + a] * pbar[i * R + b];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            Gs[a * R + b] = s;
            Gs[b * R + a] = s;
        }
    }
    __syncthreads();
    if (warp == 0) {
        factor_gram_warp<R>(Gs, Rs, Ts, drop, p.r, p.drop_tol, lane);
        double* T = p.ws.T + d.t_off;
        for (int idx = lane; idx < R * R; idx += 32) T[idx] = Ts[idx];
    }
}

// Distributed step, after the all-reduce of Q: Q_bar = sum / W_global into
// the workspace (stride R) and the caller's Q (stride r).
template <int R>
__global__ void k_dist_qbar(Params p) {
    const int l = blockIdx.y;
    const LayerDesc d = p.t.layers[l];
    float* qbar = p.ws.qbar + d.qrow_off;
    float* qout = p.t.q[l];
    const double* qsum = p.dist_in + d.qrow_off;
    const int r = p.r;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < d.n * R;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float v = static_cast<float>(qsum[idx] * p.inv_w_global);
        qbar[idx] = v;
        const int k = static_cast<int>(idx % R);
        if (k < r) qout[(idx / R) * r + k] = v;
    }
}

// ---------------------------------------------------------------------------
// Rayleigh-Ritz rotation after converged subspace iterations (SVD refresh):
// C = Q_bar^T Q_bar = W diag(lambda) W^T (cyclic Jacobi, float64, one warp,
// eigenvalues sorted descending, every column of W signed so that its
// largest-magnitude entry is positive), then P_hat <- P_hat W and
// Q_bar <- Q_bar W.  When span(P_hat) is the top-r left singular subspace of
// the worker mean, this makes P_hat = U_r and Q_bar = V_r Sigma_r; P_hat Q_bar^T
// is unchanged.  One CTA per layer.
template <int R>
__global__ void __launch_bounds__(kThreads) k_rayleigh_ritz(Params p) {
    __shared__ double C[R * R];
    __shared__ double V[R * R];
    __shared__ double Wm[R * R];
    __shared__ double lam[R];
    __shared__ int order[R];
    const int l = blockIdx.x;
    const LayerDesc d = p.t.layers[l];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = p.r;
    constexpr int NG = R * (R + 1) / 2;
    float* qbar = p.ws.qbar + d.qrow_off;
    float* phat = p.ws.phat + d.prow_off;

    // 1) C = Q_bar^T Q_bar (pairs over warps, rows over lanes, fixed order)
    for (int pidx = warp; pidx < NG; pidx += kWarps) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = 0.0;
        for (int64_t j = lane; j < d.n; j += 32)
            s += static_cast<double>(qbar[j * R + a]) * static_cast<double>(qbar[j * R + b]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            C[a * R + b] = s;
            C[b * R + a] = s;
        }
    }
    __syncthreads();

    // 2) eigen-decomposition of the r x r block by cyclic Jacobi (warp 0)
    if (warp == 0) {
        for (int idx = lane; idx < R * R; idx += 32) V[idx] = (idx / R == idx % R) ? 1.0 : 0.0;
        __syncwarp();
        double scale = 0.0;
        for (int k = 0; k < r; ++k) scale += C[k * R + k] * C[k * R + k];
        for (int sweep = 0; sweep < 40; ++sweep) {
            double off = 0.0;
            for (int a = 0; a < r; ++a)
                for (int b = a + 1; b < r; ++b) off += C[a * R + b] * C[a * R + b];
            if (!(off > 1e-30 * scale)) break;   // converged (also stops on NaN)
            for (int a = 0; a < r - 1; ++a) {
                for (int b = a + 1; b < r; ++b) {
                    const double apq = C[a * R + b];
                    if (apq == 0.0) continue;
                    const double theta = (C[b * R + b] - C[a * R + a]) / (2.0 * apq);
                    const double t = (theta == 0.0) ? 1.0
                                                    : copysign(1.0, theta) / (fabs(theta) + sqrt(theta * theta + 1.0));
                    const double c = 1.0 / sqrt(t * t + 1.0);
                    const double sn = t * c;
                    const int k = lane;
                    if (k < r) {
                        const double cp = C[k * R + a], cq = C[k * R + b];
                        C[k * R + a] = c * cp - sn * cq;
                        C[k * R + b] = sn * cp + c * cq;
                    }
                    __syncwarp();
                    if (k < r) {
                        const double rp = C[a * R + k], rq = C[b * R + k];
                        C[a * R + k] = c * rp - sn * rq;
                        C[b * R + k] = sn * rp + c * rq;
                        const double vp = V[k * R + a], vq = V[k * R + b];
                        V[k * R + a] = c * vp - sn * vq;
                        V[k * R + b] = sn * vp + c * vq;
                    }
                    __syncwarp();
                }
            }
        }
        if (lane == 0) {
            for (int k = 0; k < R; ++k) {
                lam[k] = (k < r) ? C[k * R + k] : 0.0;
                order[k] = k;
            }
            for (int a = 0; a < r; ++a) {   // selection sort, descending, stable
                int best = a;
                for (int b = a + 1; b < r; ++b)
                    if (lam[order[b]] > lam[order[best]]) best = b;
                const int tmp = order[a];
                for (int b = best; b > a; --b) order[b] = order[b - 1];
                order[a] = tmp;
            }
        }
        __syncwarp();
        for (int idx = lane; idx < R * R; idx += 32) Wm[idx] = 0.0;
        __syncwarp();
        if (lane < r) {
            const int src = order[lane];
            int arg = 0;
            double best = -1.0;
            for (int k = 0; k < r; ++k) {
                const double v = fabs(V[k * R + src]);
                if (v > best) {
                    best = v;
                    arg = k;
                }
            }
            const double sg = (V[arg * R + src] < 0.0) ? -1.0 : 1.0;
            for (int k = 0; k < r; ++k) Wm[k * R + lane] = sg * V[k * R + src];
        }
    }
    __syncthreads();

    // 3) rotate Q_bar and P_hat in place (one row per thread)
    float* qout = p.t.q[l];
    float* pout = (p.t.p_hat_out != nullptr) ? p.t.p_hat_out[l] : nullptr;
    for (int64_t j = tid; j < d.n; j += kThreads) {
        double row[R];
#pragma unroll
        for (int k = 0; k < R; ++k) row[k] = qbar[j * R + k];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            double v = 0.0;
#pragma unroll
            for (int a = 0; a < R; ++a) v += row[a] * Wm[a * R + k];
            const float f = static_cast<float>(v);
            qbar[j * R + k] = f;
            if (k < r) qout[j * r + k] = f;
        }
    }
    for (int64_t i = tid; i < d.m; i += kThreads) {
        double row[R];
#pragma unroll
        for (int k = 0; k < R; ++k) row[k] = phat[i * R + k];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            double v = 0.0;
#pragma unroll
            for (int a = 0; a < R; ++a) v += row[a] * Wm[a * R + k];
            const float f = static_cast<float>(v);
            phat[i * R + k] = f;
            if (pout != nullptr && k < r) pout[i * r + k] = f;
        }
    }
}

// ---------------------------------------------------------------------------
// small tensors: mean over workers (+ optional momentum)
__global__ void k_vec_mean(const float* const* vecs, float* const* out, const int64_t* len, int count, int W,
                           float inv_w, float* const* params, float* const* mom, float lr, float beta) {
    const int k = blockIdx.y;
    const int64_t nk = len[k];
    float* o = out[k];
    float* x = (params != nullptr) ? params[k] : nullptr;
    float* mo = (mom != nullptr) ? mom[k] : nullptr;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < nk;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float s = 0.f;
        for (int w = 0; w < W; ++w) s += vecs[w * count + k][e];
        const float g = s * inv_w;
        o[e] = g;
        if (x != nullptr && mo != nullptr) {
            const float mv = fmaf(beta, mo[e], g);
            mo[e] = mv;
            x[e] = fmaf(-lr, mv, x[e]);
        }
    }
}

// ---------------------------------------------------------------------------
// initial Q: Philox4x64-10 (Salmon et al., SC'11) + Box-Muller (1958)
struct Philox4x64 {
    static constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull;
    static constexpr uint64_t M1 = 0xCA5A826395121157ull;
    static constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull;
    static constexpr uint64_t W1 = 0xBB67AE8584CAA73Bull;
    __device__ static void run(uint64_t (&x)[4], uint64_t k0, uint64_t k1) {
#pragma unroll
        for (int rnd = 0; rnd < 10; ++rnd) {
            if (rnd) {
                k0 += W0;
                k1 += W1;
            }
            const uint64_t hi0 = __umul64hi(M0, x[0]), lo0 = M0 * x[0];
            const uint64_t hi1 = __umul64hi(M1, x[2]), lo1 = M1 * x[2];
            const uint64_t y0 = hi1 ^ x[1] ^ k0;
            const uint64_t y2 = hi0 ^ x[3] ^ k1;
            x[0] = y0;
            x[1] = lo1;
            x[2] = y2;
            x[3] = lo0;
        }
    }
};

__global__ void k_init_q(float* const* q, const LayerDesc* layers, int r, uint64_t seed, uint64_t draw) {
    const int l = blockIdx.y;
    const int64_t total = layers[l].n * r;
    const int64_t nb = (total + 3) / 4;
    float* out = q[l];
    constexpr double kTwoPi = 2.0 * 3.141592653589793;
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nb;
         b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint64_t x[4] = {static_cast<uint64_t>(b), draw, 0ull, 0ull};
        Philox4x64::run(x, seed, static_cast<uint64_t>(l));
        double z[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const double u0 = (static_cast<double>(x[2 * h] >> 11) + 0.5) * (1.0 / 9007199254740992.0);
            const double u1 = (static_cast<double>(x[2 * h + 1] >> 11) + 0.5) * (1.0 / 9007199254740992.0);
            const double rho = sqrt(-2.0 * log(u0));
            z[2 * h] = rho * cos(kTwoPi * u1);
            z[2 * h + 1] = rho * sin(kTwoPi * u1);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int64_t e = 4 * b + t;
            if (e < total) out[e] = static_cast<float>(z[t]);
        }
    }
}

}  // namespace psgd
