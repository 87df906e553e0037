// Host side of libpsgd: the C ABI declared in include/psgd.h.
//
// One context = one set of layer shapes, a rank, a worker count.  It owns
// the descriptor table, the tile map, the workspace (P partials, P_bar,
// P_hat, Gram partials, T, Q partials, Q_bar, counters, status word) and
// the device copies of the caller's pointer tables.
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cstdarg>
#include <mutex>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "psgd.h"
#include "kernels.cuh"

using psgd::LayerDesc;

namespace {

constexpr double kDropTol = 1e-12;
// An oversampled refresh stops a layer once the estimated convergence
// factor of its top-r subspace, (lambda_{r'} / lambda_r)^(iterations), is
// at most this: well below the float32 resolution of the iterates, with a
// margin for the unknown angle of the starting block.
constexpr double kRefreshEps = 1e-10;
constexpr int64_t kTileTargetElems = 65536;  // worker elements per tile (all W workers)
constexpr int kRowsFloatsMax = psgd::kRowsFloatsMax;   // TM * R bound (shared-memory rows buffer)

int pad_rank(int r) {
    int R = 1;
    while (R < r) R <<= 1;
    return R;
}

// lanes load VEC adjacent columns (a chunk is up to 32 * VEC columns); the
// lane-per-column kernels (rank <= 8) keep VEC x R values of Q per lane in
// registers, the tensor-core and wide kernels (rank 16, 32) do not
int max_vec_for_rank(int R) { return R <= 4 ? 4 : (R <= 8 ? 2 : 4); }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Element counts of one layer's share of the workspace.
struct LayerSizes {
    int64_t prow, qrow, ppart, qpart, gram, gsup, qsup, t, cnt, tiles;
};

// Tile geometry of one m x n layer at padded rank R with W workers: lane
// vector width, balanced column chunks, rows per tile for ~64K worker
// elements per tile, super-blocks for the two-level reductions.
LayerDesc layer_geometry(int64_t m, int64_t n, int R, int workers, LayerSizes* sz) {
    LayerDesc d{};
    d.m = m;
    d.n = n;
    d.vec = 1;
    for (int v : {4, 2, 1})
        if (v <= max_vec_for_rank(R) && n % v == 0) {
            d.vec = v;
            break;
        }
    d.nvec = static_cast<int>(n / d.vec);
    d.nchunk = (d.nvec + 31) / 32;
    d.slots = (d.nvec + d.nchunk - 1) / d.nchunk;
    const int64_t cols = static_cast<int64_t>(d.slots) * d.vec;
    int64_t tm = (kTileTargetElems + cols * workers - 1) / (cols * workers);
    tm = (tm + 7) / 8 * 8;
    tm = std::max<int64_t>(8, std::min<int64_t>(tm, std::min(R >= 16 ? psgd::kWideRows : 512, kRowsFloatsMax / R)));
    tm = std::min<int64_t>(tm, (m + 7) / 8 * 8);
    if (R >= 16) tm = tm <= 16 ? 16 : (tm <= 32 ? 32 : 64);   // whole 16-row groups of the tensor-core passes
    d.tm = static_cast<int>(tm);
    d.nrb = static_cast<int>((m + tm - 1) / tm);
    d.nsup = (d.nrb + psgd::kSuper - 1) / psgd::kSuper;
    const int NG = R * (R + 1) / 2;
    sz->prow = m * R;
    sz->qrow = n * R;
    sz->ppart = static_cast<int64_t>(d.nchunk) * m * R;
    sz->qpart = static_cast<int64_t>(d.nrb) * n * R;
    sz->gram = static_cast<int64_t>(d.nrb) * NG;
    sz->gsup = static_cast<int64_t>(d.nsup) * NG;
    sz->qsup = static_cast<int64_t>(d.nsup) * n * R;
    sz->t = static_cast<int64_t>(R) * R;
    sz->cnt = psgd::counter_layout(d.nrb, d.nsup, d.nchunk).total;
    sz->tiles = static_cast<int64_t>(d.nrb) * d.nchunk;
    return d;
}

// Device copy of a host pointer table.  Re-uploaded only when the contents
// change; uploads go through a small ring of pinned buffers so that an
// upload never overwrites a host buffer a previous async copy still reads.
class DevTable {
public:
    ~DevTable() { release(); }
    void release() {
        if (dev_) cudaFree(dev_);
        for (int i = 0; i < kRing; ++i) {
            if (ring_[i]) cudaFreeHost(ring_[i]);
            if (ev_[i]) cudaEventDestroy(ev_[i]);
            ring_[i] = nullptr;
            ev_[i] = nullptr;
        }
        dev_ = nullptr;
        cap_ = 0;
        cache_.clear();
        valid_ = false;
    }
    cudaError_t reserve(size_t words) {
        if (dev_ && words <= cap_) return cudaSuccess;
        release();
        cudaError_t e = cudaMalloc(&dev_, std::max<size_t>(words, 1) * 8);
        if (e != cudaSuccess) return e;
        for (int i = 0; i < kRing; ++i) {
            e = cudaMallocHost(&ring_[i], std::max<size_t>(words, 1) * 8);
            if (e != cudaSuccess) return e;
            e = cudaEventCreateWithFlags(&ev_[i], cudaEventDisableTiming);
            if (e != cudaSuccess) return e;
        }
        cap_ = words;
        return cudaSuccess;
    }
    // Returns cudaSuccess and uploads (on stream) when vals differ.
    cudaError_t update(const std::vector<uint64_t>& vals, cudaStream_t stream) {
        cudaError_t e = reserve(vals.size());
        if (e != cudaSuccess) return e;
        if (valid_ && vals == cache_) return cudaSuccess;
        const int slot = next_;
        next_ = (next_ + 1) % kRing;
        e = cudaEventSynchronize(ev_[slot]);  // normally long complete
        if (e != cudaSuccess) return e;
        if (!vals.empty()) std::memcpy(ring_[slot], vals.data(), vals.size() * 8);
        if (!vals.empty()) {
            e = cudaMemcpyAsync(dev_, ring_[slot], vals.size() * 8, cudaMemcpyHostToDevice, stream);
            if (e != cudaSuccess) return e;
        }
        e = cudaEventRecord(ev_[slot], stream);
        if (e != cudaSuccess) return e;
        cache_ = vals;
        valid_ = true;
        return cudaSuccess;
    }
    void* dev() const { return dev_; }

private:
    static constexpr int kRing = 4;
    void* dev_ = nullptr;
    void* ring_[kRing] = {nullptr, nullptr, nullptr, nullptr};
    cudaEvent_t ev_[kRing] = {nullptr, nullptr, nullptr, nullptr};
    int next_ = 0;
    size_t cap_ = 0;
    std::vector<uint64_t> cache_;
    bool valid_ = false;
};

thread_local std::string g_create_error;

}  // namespace

struct psgd_ctx {
    int device = 0;
    int L = 0, W = 0, r = 0, R = 0;
    int dtype = PSGD_F32;
    unsigned flags = 0;
    uint64_t seed = 0;
    std::vector<psgd_layer> shapes;
    std::vector<LayerDesc> desc;
    int64_t ntiles = 0;
    size_t smem_a = 0, smem_b = 0, smem_c = 0;

    // device allocations
    void* ws = nullptr;
    size_t ws_bytes = 0;
    LayerDesc* desc_d = nullptr;
    int* tile_layer_d = nullptr;
    psgd::Work work{};

    DevTable tab_w;    // grads[W*L], errors[W*L]
    DevTable tab_l;    // q[L], p_hat[L], recon[L]
    DevTable tab_m;    // params[L], mom[L]
    DevTable tab_e;    // errors[W*L] for materialisation
    DevTable tab_v;    // vector tables
    DevTable tab_q;    // q[L] for the initial draw

    void* stage = nullptr;  // device staging of host gradients
    size_t stage_bytes = 0;
    // host-buffer steps: the uploads run on their own stream, one event per
    // layer group, so that a group's passes start once its bytes are in
    cudaStream_t up_stream = nullptr;
    cudaEvent_t up_start = nullptr;
    std::vector<cudaEvent_t> up_ev;

    // optional per-kernel timing (psgd_profile_*)
    bool profiling = false;
    std::vector<std::array<cudaEvent_t, 6>> prof_ev;   // begin/end of passes A, B, C
    size_t prof_used = 0;

    int iters = 1;          // power iterations per step
    int stall_products = 0; // psgd_test_stall_products
    int w_global = 0;       // workers over all ranks (distributed step); 0 = W
    int dist_phase = 0;     // distributed step: 0 idle, 1 after P, 2 after Q
    bool tab_l_has_recon = false;
    cudaEvent_t* dist_ev = nullptr;   // profiling events of the step in progress
    int svd_every = 0;      // SVD refresh period in steps (0: off)
    int svd_iters = 0;      // subspace iterations on a refresh step (the cap)
    int svd_over = 8;       // oversampling columns of a refresh step
    psgd_ctx* sub = nullptr;   // rank r + p context iterated on refresh steps
    float* qsub = nullptr;     // its Q block per layer (n x (r + p)), one allocation
    DevTable tab_sub;          // q' table | L null p_hat | L null recon
    std::vector<uint64_t> tab_sub_vals;
    uint64_t steps_done = 0;

    bool have_step = false;
    bool errors_hold_m = false;
    cudaStream_t last_stream = nullptr;
    std::string err;
};

namespace {

int fail(psgd_ctx* ctx, int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    if (ctx)
        ctx->err = buf;
    else
        g_create_error = buf;
    return code;
}

int cuda_fail(psgd_ctx* ctx, cudaError_t e, const char* what) {
    return fail(ctx, PSGD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Keeps the caller's current device: switches to the context's device for
// the duration of a call.
struct DeviceGuard {
    int prev = -1;
    bool switched = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
            switched = (cudaSetDevice(dev) == cudaSuccess);
        }
    }
    ~DeviceGuard() {
        if (switched) cudaSetDevice(prev);
    }
};

// ---- kernel dispatch over the padded rank ---------------------------------

template <int R>
struct Launch {
    static void* pass_a(int dtype, bool lazy, bool sf) {
        if (dtype == PSGD_BF16) {
            if (lazy) return sf ? (void*)psgd::k_pass_a<R, uint16_t, true, true, false> : (void*)psgd::k_pass_a<R, uint16_t, true, false, false>;
            return sf ? (void*)psgd::k_pass_a<R, uint16_t, false, true, false> : (void*)psgd::k_pass_a<R, uint16_t, false, false, false>;
        }
        if (lazy) return sf ? (void*)psgd::k_pass_a<R, float, true, true, false> : (void*)psgd::k_pass_a<R, float, true, false, false>;
        return sf ? (void*)psgd::k_pass_a<R, float, false, true, false> : (void*)psgd::k_pass_a<R, float, false, false, false>;
    }
    // later power iterations: M already formed in the error buffers
    static void* pass_a_m(bool sf) {
        return sf ? (void*)psgd::k_pass_a<R, float, false, true, true> : (void*)psgd::k_pass_a<R, float, false, false, true>;
    }
    static void* pass_b(bool sf) { return sf ? (void*)psgd::k_pass_b<R, true> : (void*)psgd::k_pass_b<R, false>; }
    static void* pass_c() { return (void*)psgd::k_pass_c<R>; }
    static void* rayleigh_ritz() { return (void*)psgd::k_rayleigh_ritz<R>; }
    static void* dist_orth() { return (void*)psgd::k_dist_orth<R>; }
    static void* dist_qbar() { return (void*)psgd::k_dist_qbar<R>; }
    static void* phat() { return (void*)psgd::k_phat<R>; }
};

void* kernel_ptr(int which, int R, int dtype, bool lazy, bool sf) {
#define PSGD_CASE(RR)                                        \
    case RR:                                                 \
        if (which == 0) return Launch<RR>::pass_a(dtype, lazy, sf); \
        if (which == 1) return Launch<RR>::pass_b(sf);       \
        if (which == 3) return Launch<RR>::pass_a_m(sf);     \
        if (which == 4) return Launch<RR>::rayleigh_ritz();  \
        if (which == 5) return Launch<RR>::dist_orth();      \
        if (which == 6) return Launch<RR>::dist_qbar();      \
        if (which == 7) return Launch<RR>::phat();           \
        return Launch<RR>::pass_c();
    switch (R) {
        PSGD_CASE(1)
        PSGD_CASE(2)
        PSGD_CASE(4)
        PSGD_CASE(8)
        PSGD_CASE(16)
        PSGD_CASE(32)
        default:
            return nullptr;
    }
#undef PSGD_CASE
}

size_t smem_need(int which, int R, int W, int tm, int vec, bool lazy = false) {
#define PSGD_CASE(RR)                                                         \
    case RR:                                                                  \
        if (which == 0 || which == 3) return psgd::SmemA<RR>::total(W, tm, lazy); \
        if (which == 1) return psgd::SmemB<RR>::total(W, tm, vec);            \
        return psgd::SmemC<RR>::total(W, tm);
    switch (R) {
        PSGD_CASE(1)
        PSGD_CASE(2)
        PSGD_CASE(4)
        PSGD_CASE(8)
        PSGD_CASE(16)
        PSGD_CASE(32)
        default:
            return 0;
    }
#undef PSGD_CASE
}

psgd::Params base_params(psgd_ctx* ctx) {
    psgd::Params p{};
    p.t.layers = ctx->desc_d;
    p.t.tile_layer = ctx->tile_layer_d;
    p.ws = ctx->work;
    p.num_layers = ctx->L;
    p.workers = ctx->W;
    p.r = ctx->r;
    p.inv_w = 1.0f / static_cast<float>(ctx->W);
    p.drop_tol = kDropTol;
    p.inv_w_global = 1.0 / static_cast<double>(ctx->w_global > 0 ? ctx->w_global : ctx->W);
    p.stall_products = ctx->stall_products;
    return p;
}

// Grid of k_phat: (x, L), x covering the largest layer's m R elements
// (grid-stride beyond 4096 blocks).
dim3 phat_grid(int64_t maxm, size_t num_layers, int R) {
    const int64_t gx = std::min<int64_t>(4096, (std::max<int64_t>(1, maxm) * R + psgd::kThreads - 1) / psgd::kThreads);
    return dim3(static_cast<unsigned>(std::max<int64_t>(1, gx)), static_cast<unsigned>(num_layers));
}
dim3 phat_grid(const std::vector<LayerDesc>& desc, int R) {
    int64_t maxm = 1;
    for (auto& d : desc) maxm = std::max(maxm, d.m);
    return phat_grid(maxm, desc.size(), R);
}

// The second pass (which == 1) is preceded by k_phat, which forms P_hat
// from P_bar and T once per layer.
int launch(psgd_ctx* ctx, int which, bool lazy, const psgd::Params& p, size_t smem, cudaStream_t stream) {
    if (ctx->ntiles == 0) return PSGD_OK;
    void* fn = kernel_ptr(which, ctx->R, ctx->dtype, lazy, (ctx->flags & PSGD_FLAG_SUM_FIRST) != 0);
    if (!fn) return fail(ctx, PSGD_ERR_ARG, "no kernel for rank %d", ctx->r);
    void* args[] = {const_cast<psgd::Params*>(&p)};
    if (which == 1) {
        cudaError_t e = cudaLaunchKernel(kernel_ptr(7, ctx->R, ctx->dtype, false, false), phat_grid(ctx->desc, ctx->R),
                                         dim3(psgd::kThreads), args, 0, stream);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "P_hat launch");
    }
    cudaError_t e = cudaLaunchKernel(fn, dim3(static_cast<unsigned>(ctx->ntiles)), dim3(psgd::kThreads), args, smem,
                                     stream);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "kernel launch");
    return PSGD_OK;
}

// launch() over the layers [l0, l1) only: their tiles are one contiguous
// range of the grouped grid, and the P_hat grid covers just those layers.
int launch_layers(psgd_ctx* ctx, int which, bool lazy, const psgd::Params& p0, size_t smem, cudaStream_t stream,
                  int l0, int l1) {
    const LayerDesc& last = ctx->desc[l1 - 1];
    const int64_t t0 = ctx->desc[l0].tile_begin;
    const int64_t t1 = last.tile_begin + static_cast<int64_t>(last.nrb) * last.nchunk;
    if (t1 <= t0) return PSGD_OK;
    void* fn = kernel_ptr(which, ctx->R, ctx->dtype, lazy, (ctx->flags & PSGD_FLAG_SUM_FIRST) != 0);
    if (!fn) return fail(ctx, PSGD_ERR_ARG, "no kernel for rank %d", ctx->r);
    psgd::Params p = p0;
    p.tile_base = static_cast<int>(t0);
    p.layer_base = l0;
    void* args[] = {&p};
    if (which == 1) {
        int64_t maxm = 1;
        for (int l = l0; l < l1; ++l) maxm = std::max(maxm, ctx->desc[l].m);
        cudaError_t e = cudaLaunchKernel(kernel_ptr(7, ctx->R, ctx->dtype, false, false),
                                         phat_grid(maxm, static_cast<size_t>(l1 - l0), ctx->R), dim3(psgd::kThreads),
                                         args, 0, stream);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "P_hat launch");
    }
    cudaError_t e = cudaLaunchKernel(fn, dim3(static_cast<unsigned>(t1 - t0)), dim3(psgd::kThreads), args, smem, stream);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "kernel launch");
    return PSGD_OK;
}

// Layer groups of a host-buffer step: contiguous layer ranges of about
// equal size, at most kUploadGroups of them.  Group g's passes wait only
// for group g's upload, so the later groups' copies overlap them.
constexpr int kUploadGroups = 8;
using LayerGroups = std::vector<std::pair<int, int>>;
LayerGroups upload_groups(const psgd_ctx* ctx) {
    LayerGroups g;
    double total = 0.0;
    for (auto& d : ctx->desc) total += static_cast<double>(d.m) * static_cast<double>(d.n);
    const int K = std::min(ctx->L, kUploadGroups);
    double acc = 0.0;
    int start = 0;
    for (int l = 0; l < ctx->L; ++l) {
        acc += static_cast<double>(ctx->desc[l].m) * static_cast<double>(ctx->desc[l].n);
        const bool cut = static_cast<int>(g.size()) < K - 1 && acc >= total * static_cast<double>(g.size() + 1) / K;
        if (cut || l == ctx->L - 1) {
            g.emplace_back(start, l + 1);
            start = l + 1;
        }
    }
    return g;
}

// The upload stream and one event per group; the uploads start after
// everything already queued on the caller's stream (the previous step's
// passes may still read the staging).
int begin_upload(psgd_ctx* ctx, size_t groups, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    if (!ctx->up_stream) e = cudaStreamCreateWithFlags(&ctx->up_stream, cudaStreamNonBlocking);
    if (e == cudaSuccess && !ctx->up_start) e = cudaEventCreateWithFlags(&ctx->up_start, cudaEventDisableTiming);
    while (e == cudaSuccess && ctx->up_ev.size() < groups) {
        cudaEvent_t x = nullptr;
        e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
        if (e == cudaSuccess) ctx->up_ev.push_back(x);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ctx->up_start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->up_stream, ctx->up_start, 0);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "upload stream");
    return PSGD_OK;
}

int check_ptr_array(psgd_ctx* ctx, const void* const* a, size_t count, bool allow_null_entries, const char* name) {
    if (count && !a) return fail(ctx, PSGD_ERR_ARG, "%s: null pointer array", name);
    for (size_t i = 0; i < count; ++i) {
        if (!a[i]) {
            if (allow_null_entries) continue;
            return fail(ctx, PSGD_ERR_ARG, "%s[%zu] is null", name, i);
        }
        if (!aligned16(a[i])) return fail(ctx, PSGD_ERR_ALIGN, "%s[%zu] is not 16-byte aligned", name, i);
    }
    return PSGD_OK;
}

}  // namespace

extern "C" {

const char* psgd_last_error(const psgd_ctx* ctx) { return ctx ? ctx->err.c_str() : g_create_error.c_str(); }

int psgd_create(psgd_ctx** out, const psgd_layer* layers, int num_layers, int rank, int workers, uint64_t seed,
                int grad_dtype, unsigned flags) {
    g_create_error.clear();
    if (!out) return fail(nullptr, PSGD_ERR_ARG, "out is null");
    *out = nullptr;
    if (num_layers < 0 || (num_layers > 0 && !layers)) return fail(nullptr, PSGD_ERR_ARG, "bad layer list");
    if (rank < 1 || rank > psgd::kMaxRank) return fail(nullptr, PSGD_ERR_ARG, "rank %d not in [1, 32]", rank);
    if (workers < 1 || workers > psgd::kMaxWorkers)
        return fail(nullptr, PSGD_ERR_ARG, "workers %d not in [1, %d]", workers, psgd::kMaxWorkers);
    if (grad_dtype != PSGD_F32 && grad_dtype != PSGD_BF16) return fail(nullptr, PSGD_ERR_ARG, "bad grad dtype");
    if (flags & ~(PSGD_FLAG_LAZY_ERRORS | PSGD_FLAG_SUM_FIRST | PSGD_FLAG_NO_WARM_START))
        return fail(nullptr, PSGD_ERR_ARG, "unknown flags");
    for (int l = 0; l < num_layers; ++l) {
        const int64_t m = layers[l].m, n = layers[l].n;
        if (m < 1 || n < 1) return fail(nullptr, PSGD_ERR_ARG, "layer %d: shape %lld x %lld", l, (long long)m, (long long)n);
        if (rank > m || rank > n)
            return fail(nullptr, PSGD_ERR_ARG, "layer %d: rank %d > min(%lld, %lld)", l, rank, (long long)m, (long long)n);
        if (m > (int64_t(1) << 31) || n > (int64_t(1) << 31) || m * n > (int64_t(1) << 40))
            return fail(nullptr, PSGD_ERR_ARG, "layer %d too large", l);
    }

    psgd_ctx* ctx = new psgd_ctx();
    cudaGetDevice(&ctx->device);
    ctx->L = num_layers;
    ctx->W = workers;
    ctx->r = rank;
    ctx->R = pad_rank(rank);
    ctx->dtype = grad_dtype;
    ctx->flags = flags;
    ctx->seed = seed;
    ctx->shapes.assign(layers, layers + num_layers);

    const int R = ctx->R;
    int64_t tiles = 0, prow = 0, qrow = 0, ppart = 0, qpart = 0, gram = 0, gsup = 0, qsup = 0, tt = 0, cnt = 0;
    std::vector<int> tile_layer;
    for (int l = 0; l < num_layers; ++l) {
        LayerSizes sz{};
        LayerDesc d = layer_geometry(layers[l].m, layers[l].n, R, workers, &sz);
        d.tile_begin = tiles;
        d.prow_off = prow;
        d.qrow_off = qrow;
        d.ppart_off = ppart;
        d.qpart_off = qpart;
        d.gram_off = gram;
        d.gsup_off = gsup;
        d.qsup_off = qsup;
        d.t_off = tt;
        d.cnt_off = cnt;
        tiles += sz.tiles;
        prow += sz.prow;
        qrow += sz.qrow;
        ppart += sz.ppart;
        qpart += sz.qpart;
        gram += sz.gram;
        gsup += sz.gsup;
        qsup += sz.qsup;
        tt += sz.t;
        cnt += sz.cnt;
        for (int64_t t = 0; t < sz.tiles; ++t) tile_layer.push_back(l);
        ctx->desc.push_back(d);
        ctx->smem_a = std::max(ctx->smem_a, smem_need(0, R, workers, d.tm, d.vec, (flags & PSGD_FLAG_LAZY_ERRORS) != 0));
        ctx->smem_b = std::max(ctx->smem_b, smem_need(1, R, workers, d.tm, d.vec));
        ctx->smem_c = std::max(ctx->smem_c, smem_need(2, R, workers, d.tm, d.vec));
    }
    if (tiles > 0x7fffffff) {
        delete ctx;
        return fail(nullptr, PSGD_ERR_ARG, "too many tiles");
    }
    ctx->ntiles = tiles;

    // one workspace allocation, carved into 256-byte aligned pieces
    size_t off = 0;
    auto carve = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + std::max<size_t>(bytes, 1), 256);
        return o;
    };
    const size_t o_desc = carve(sizeof(LayerDesc) * std::max(1, num_layers));
    const size_t o_tile = carve(sizeof(int) * std::max<int64_t>(1, tiles));
    const size_t o_pbar = carve(sizeof(double) * prow);
    const size_t o_phat = carve(sizeof(float) * prow);
    const size_t o_qbar = carve(sizeof(float) * qrow);
    const size_t o_ppart = carve(sizeof(double) * ppart);
    const size_t o_qpart = carve(sizeof(double) * qpart);
    const size_t o_gram = carve(sizeof(double) * gram);
    const size_t o_gsup = carve(sizeof(double) * gsup);
    const size_t o_qsup = carve(sizeof(double) * qsup);
    const size_t o_T = carve(sizeof(double) * tt);
    const size_t o_cnt = carve(sizeof(unsigned) * cnt);
    const size_t o_status = carve(sizeof(int));
    const size_t o_conv = carve(sizeof(int) * std::max(1, num_layers));
    ctx->ws_bytes = off;
    cudaError_t e = cudaMalloc(&ctx->ws, ctx->ws_bytes);
    if (e != cudaSuccess) {
        fail(nullptr, PSGD_ERR_OOM, "workspace of %zu bytes: %s", ctx->ws_bytes, cudaGetErrorString(e));
        delete ctx;
        return PSGD_ERR_OOM;
    }
    unsigned char* base = static_cast<unsigned char*>(ctx->ws);
    ctx->desc_d = reinterpret_cast<LayerDesc*>(base + o_desc);
    ctx->tile_layer_d = reinterpret_cast<int*>(base + o_tile);
    ctx->work.pbar = reinterpret_cast<double*>(base + o_pbar);
    ctx->work.phat = reinterpret_cast<float*>(base + o_phat);
    ctx->work.qbar = reinterpret_cast<float*>(base + o_qbar);
    ctx->work.ppart = reinterpret_cast<double*>(base + o_ppart);
    ctx->work.qpart = reinterpret_cast<double*>(base + o_qpart);
    ctx->work.gram = reinterpret_cast<double*>(base + o_gram);
    ctx->work.gsup = reinterpret_cast<double*>(base + o_gsup);
    ctx->work.qsup = reinterpret_cast<double*>(base + o_qsup);
    ctx->work.T = reinterpret_cast<double*>(base + o_T);
    ctx->work.cnt = reinterpret_cast<unsigned*>(base + o_cnt);
    ctx->work.status = reinterpret_cast<int*>(base + o_status);
    ctx->work.conv_iter = reinterpret_cast<int*>(base + o_conv);

    e = cudaMemset(ctx->ws, 0, ctx->ws_bytes);
    if (e == cudaSuccess && num_layers > 0)
        e = cudaMemcpy(ctx->desc_d, ctx->desc.data(), sizeof(LayerDesc) * num_layers, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && tiles > 0)
        e = cudaMemcpy(ctx->tile_layer_d, tile_layer.data(), sizeof(int) * tiles, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        fail(nullptr, PSGD_ERR_CUDA, "workspace init: %s", cudaGetErrorString(e));
        cudaFree(ctx->ws);
        delete ctx;
        return PSGD_ERR_CUDA;
    }
    // opt in to the dynamic shared memory each kernel of this context needs.
    // The attribute is per kernel, shared by every context: only ever raise
    // it, so that a context with smaller tiles never breaks an existing one.
    auto raise_smem = [](const void* fn, size_t need) -> cudaError_t {
        cudaFuncAttributes fa{};
        cudaError_t err = cudaFuncGetAttributes(&fa, fn);
        if (err != cudaSuccess) return err;
        if (static_cast<size_t>(fa.maxDynamicSharedSizeBytes) >= need) return cudaSuccess;
        return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(need));
    };
    for (int lazy = 0; lazy < 2; ++lazy) {
        const bool sf = (flags & PSGD_FLAG_SUM_FIRST) != 0;
        const void* fa = kernel_ptr(0, R, grad_dtype, lazy != 0, sf);
        const void* fb = kernel_ptr(1, R, grad_dtype, lazy != 0, sf);
        const void* fc = kernel_ptr(2, R, grad_dtype, lazy != 0, sf);
        const void* fam = kernel_ptr(3, R, grad_dtype, false, sf);
        e = raise_smem(fa, ctx->smem_a);
        if (e == cudaSuccess) e = raise_smem(fam, ctx->smem_a);
        if (e == cudaSuccess) e = raise_smem(fb, ctx->smem_b);
        if (e == cudaSuccess) e = raise_smem(fc, ctx->smem_c);
        if (e != cudaSuccess) {
            fail(nullptr, PSGD_ERR_CUDA, "shared-memory opt-in: %s", cudaGetErrorString(e));
            cudaFree(ctx->ws);
            delete ctx;
            return PSGD_ERR_CUDA;
        }
    }
    *out = ctx;
    return PSGD_OK;
}

void psgd_destroy(psgd_ctx* ctx) {
    if (!ctx) return;
    DeviceGuard g(ctx->device);
    cudaDeviceSynchronize();
    if (ctx->sub) psgd_destroy(ctx->sub);
    if (ctx->qsub) cudaFree(ctx->qsub);
    ctx->tab_sub.release();
    if (ctx->ws) cudaFree(ctx->ws);
    if (ctx->stage) cudaFree(ctx->stage);
    for (auto& x : ctx->up_ev) cudaEventDestroy(x);
    if (ctx->up_start) cudaEventDestroy(ctx->up_start);
    if (ctx->up_stream) cudaStreamDestroy(ctx->up_stream);
    ctx->tab_w.release();
    ctx->tab_l.release();
    ctx->tab_m.release();
    ctx->tab_e.release();
    ctx->tab_v.release();
    ctx->tab_q.release();
    for (auto& a : ctx->prof_ev)
        for (auto& x : a) cudaEventDestroy(x);
    delete ctx;
}

int psgd_workspace_bytes(const psgd_ctx* ctx, size_t* bytes) {
    if (!ctx || !bytes) return PSGD_ERR_ARG;
    *bytes = ctx->ws_bytes;
    return PSGD_OK;
}

int psgd_step_launches(const psgd_ctx* ctx) {
    if (!ctx) return -1;
    if (ctx->ntiles == 0) return 0;
    int n = 3 * ctx->iters + ((ctx->flags & PSGD_FLAG_LAZY_ERRORS) ? 0 : 1);
    if (ctx->flags & PSGD_FLAG_NO_WARM_START) n += 1;
    return n;
}

int psgd_init_q(psgd_ctx* ctx, float* const* q, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    int rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(q), ctx->L, false, "q");
    if (rc) return rc;
    if (ctx->L == 0) return PSGD_OK;
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::vector<uint64_t> tab(ctx->L, 0);
    for (int l = 0; l < ctx->L; ++l) tab[l] = reinterpret_cast<uint64_t>(q[l]);
    cudaError_t e = ctx->tab_q.update(tab, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "table upload");
    int64_t maxn = 0;
    for (auto& d : ctx->desc) maxn = std::max(maxn, d.n);
    const int64_t blocks4 = (maxn * ctx->r + 3) / 4;
    const unsigned gx = static_cast<unsigned>(std::min<int64_t>(1024, (blocks4 + 255) / 256));
    psgd::k_init_q<<<dim3(std::max(1u, gx), ctx->L), 256, 0, s>>>(static_cast<float* const*>(ctx->tab_q.dev()),
                                                                  ctx->desc_d, ctx->r, ctx->seed, 0ull);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "init_q launch");
    ctx->last_stream = s;
    return PSGD_OK;
}

// Next set of profiling events (begin/end of passes A, B, C), or null when
// profiling is off.
static cudaEvent_t* profile_events(psgd_ctx* ctx, cudaError_t* err) {
    *err = cudaSuccess;
    if (!ctx->profiling) return nullptr;
    if (ctx->prof_used == ctx->prof_ev.size()) {
        std::array<cudaEvent_t, 6> a{};
        for (auto& x : a) {
            *err = cudaEventCreate(&x);
            if (*err != cudaSuccess) return nullptr;
        }
        ctx->prof_ev.push_back(a);
    }
    return ctx->prof_ev[ctx->prof_used++].data();
}

// A PowerSGD+ refresh step with an oversampled block ("From PowerSGD to
// PowerSGD+", Abstract: the projection subspace is re-aligned through an
// SVD): subspace iterations on r' = r + p columns in the rank-r' context
// ctx->sub, starting from Q' = [warm-start Q | fresh draws], each layer
// stopping once its convergence bound is met (at most svd_iters
// iterations); then Rayleigh-Ritz keeps the top r directions in this
// context's workspace and the caller's Q and P_hat.  The first iteration
// forms M = G + E over the error buffers (in lazy mode after the previous
// step's E' has been written out), so that pass C can follow as usual.
static int refresh_oversampled(psgd_ctx* ctx, const psgd::Params& p, bool lazy, cudaStream_t s, cudaEvent_t* ev) {
    psgd_ctx* sub = ctx->sub;
    int rc = PSGD_OK;
    if (lazy && ctx->errors_hold_m) {
        psgd::Params pm = p;
        pm.use_prev = 0;
        pm.do_resid = 1;
        rc = launch(ctx, 2, true, pm, ctx->smem_c, s);
        if (rc) return rc;
    }
    cudaError_t e = ctx->tab_sub.update(ctx->tab_sub_vals, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "table upload");
    float* const* qs = static_cast<float* const*>(ctx->tab_sub.dev());
    int64_t maxn = 0;
    for (auto& d : ctx->desc) maxn = std::max(maxn, d.n);
    const unsigned gx = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(1024, (maxn * sub->r + 255) / 256)));
    psgd::k_assemble_q<<<dim3(gx, ctx->L), 256, 0, s>>>(qs, p.t.q, ctx->desc_d, ctx->r, sub->r, ctx->seed,
                                                        (uint64_t(1) << 62) | (ctx->steps_done + 1));
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaMemsetAsync(sub->work.conv_iter, 0x7f, sizeof(int) * ctx->L, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "refresh set-up");

    psgd::Params ps = base_params(sub);
    ps.t.grads = p.t.grads;
    ps.t.errors = p.t.errors;
    ps.t.q = qs;
    ps.t.p_hat_out = qs + ctx->L;     // null entries: the block's P_hat stays inside
    ps.t.recon_out = qs + 2 * ctx->L;
    ps.track_conv = 1;
    ps.r_conv = ctx->r;
    ps.conv_eps = kRefreshEps;
    for (int it = 1; it <= ctx->svd_iters && !rc; ++it) {
        ps.iter = it;
        rc = launch(sub, it == 1 ? 0 : 3, false, ps, sub->smem_a, s);
        if (it == 1 && ev) {
            cudaEventRecord(ev[1], s);
            cudaEventRecord(ev[2], s);
        }
        if (!rc) rc = launch(sub, 1, false, ps, sub->smem_b, s);
    }
    if (rc) return fail(ctx, rc, "refresh iterations: %s", sub->err.c_str());
    void* fn = kernel_ptr(4, sub->R, sub->dtype, false, false);
    psgd::RRDst dst{ctx->desc_d, ctx->work.phat, ctx->work.qbar, p.t.q, p.t.p_hat_out, ctx->R, ctx->r};
    void* args[] = {&ps, &dst};
    e = cudaLaunchKernel(fn, dim3(static_cast<unsigned>(ctx->L)), dim3(psgd::kThreads), args, 0, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "Rayleigh-Ritz launch");
    if (ev) {
        cudaEventRecord(ev[3], s);
        cudaEventRecord(ev[4], s);
    }
    return PSGD_OK;
}

// With `groups` (host-buffer steps), the gradients of group g are ready
// once ctx->up_ev[g] has fired; a step that cannot run group by group
// (power iterations, refresh, profiling) waits for the whole upload.
static int step_impl(psgd_ctx* ctx, const void* const* grads, float* const* errors, float* const* q,
                     float* const* p_hat, float* const* recon, cudaStream_t s, const LayerGroups* groups = nullptr) {
    const size_t WL = static_cast<size_t>(ctx->W) * ctx->L;
    std::vector<uint64_t> tw(2 * WL);
    for (size_t i = 0; i < WL; ++i) {
        tw[i] = reinterpret_cast<uint64_t>(grads[i]);
        tw[WL + i] = reinterpret_cast<uint64_t>(errors[i]);
    }
    std::vector<uint64_t> tl(3 * ctx->L, 0);
    for (int l = 0; l < ctx->L; ++l) {
        tl[l] = reinterpret_cast<uint64_t>(q[l]);
        tl[ctx->L + l] = p_hat ? reinterpret_cast<uint64_t>(p_hat[l]) : 0;
        tl[2 * ctx->L + l] = recon ? reinterpret_cast<uint64_t>(recon[l]) : 0;
    }
    cudaError_t e = ctx->tab_w.update(tw, s);
    if (e == cudaSuccess) e = ctx->tab_l.update(tl, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "table upload");

    const bool lazy = (ctx->flags & PSGD_FLAG_LAZY_ERRORS) != 0;
    psgd::Params p = base_params(ctx);
    void* const* wt = static_cast<void* const*>(ctx->tab_w.dev());
    void* const* lt = static_cast<void* const*>(ctx->tab_l.dev());
    p.t.grads = reinterpret_cast<const void* const*>(wt);
    p.t.errors = reinterpret_cast<float* const*>(wt + WL);
    p.t.q = reinterpret_cast<float* const*>(lt);
    p.t.p_hat_out = reinterpret_cast<float* const*>(lt + ctx->L);
    p.t.recon_out = reinterpret_cast<float* const*>(lt + 2 * ctx->L);
    p.use_prev = (lazy && ctx->errors_hold_m) ? 1 : 0;

    cudaEvent_t* ev = profile_events(ctx, &e);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "profiling event");
    if (ev) cudaEventRecord(ev[0], s);
    int rc = PSGD_OK;
    if (ctx->flags & PSGD_FLAG_NO_WARM_START) {
        // no warm start: a fresh Q for this step (draw index = step number)
        int64_t maxn = 0;
        for (auto& d : ctx->desc) maxn = std::max(maxn, d.n);
        const int64_t blocks4 = (maxn * ctx->r + 3) / 4;
        const unsigned gx = static_cast<unsigned>(std::min<int64_t>(1024, (blocks4 + 255) / 256));
        psgd::k_init_q<<<dim3(std::max(1u, gx), ctx->L), 256, 0, s>>>(p.t.q, ctx->desc_d, ctx->r, ctx->seed,
                                                                      ctx->steps_done + 1);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(ctx, e, "fresh Q launch");
    }
    const bool refresh = ctx->svd_every > 0 && (ctx->steps_done + 1) % ctx->svd_every == 0;
    const bool grouped = groups && !groups->empty() && !refresh && ctx->iters == 1 && !ev;
    if (groups && !groups->empty() && !grouped) {
        e = cudaStreamWaitEvent(s, ctx->up_ev[groups->size() - 1], 0);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "upload wait");
    }
    if (grouped) {
        for (size_t g = 0; g < groups->size() && !rc; ++g) {
            const int l0 = (*groups)[g].first, l1 = (*groups)[g].second;
            e = cudaStreamWaitEvent(s, ctx->up_ev[g], 0);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "upload wait");
            rc = launch_layers(ctx, 0, lazy, p, ctx->smem_a, s, l0, l1);
            if (!rc) rc = launch_layers(ctx, 1, lazy, p, ctx->smem_b, s, l0, l1);
            if (!rc && (!lazy || recon)) {
                psgd::Params pc = p;
                pc.do_resid = lazy ? 0 : 1;
                pc.do_recon = recon ? 1 : 0;
                rc = launch_layers(ctx, 2, lazy, pc, ctx->smem_c, s, l0, l1);
            }
        }
    } else if (refresh && ctx->sub) {
        rc = refresh_oversampled(ctx, p, lazy, s, ev);
    } else {
        rc = launch(ctx, 0, lazy, p, ctx->smem_a, s);
        if (ev) {
            cudaEventRecord(ev[1], s);
            cudaEventRecord(ev[2], s);
        }
        if (!rc) rc = launch(ctx, 1, lazy, p, ctx->smem_b, s);
        const int iters = refresh ? ctx->svd_iters : ctx->iters;
        for (int it = 1; it < iters && !rc; ++it) {
            psgd::Params pi = p;
            pi.use_prev = 0;
            rc = launch(ctx, 3, false, pi, ctx->smem_a, s);
            if (!rc) rc = launch(ctx, 1, lazy, pi, ctx->smem_b, s);
        }
        if (refresh && !rc) {
            // Rayleigh-Ritz in place: one CTA per layer
            void* fn = kernel_ptr(4, ctx->R, ctx->dtype, false, false);
            psgd::RRDst dst{ctx->desc_d, ctx->work.phat, ctx->work.qbar, p.t.q, p.t.p_hat_out, ctx->R, ctx->r};
            void* args[] = {&p, &dst};
            e = cudaLaunchKernel(fn, dim3(static_cast<unsigned>(ctx->L)), dim3(psgd::kThreads), args, 0, s);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "Rayleigh-Ritz launch");
        }
        if (ev) {
            cudaEventRecord(ev[3], s);
            cudaEventRecord(ev[4], s);
        }
    }
    if (!rc && !grouped && (!lazy || recon)) {
        psgd::Params pc = p;
        pc.do_resid = lazy ? 0 : 1;
        pc.do_recon = recon ? 1 : 0;
        rc = launch(ctx, 2, lazy, pc, ctx->smem_c, s);
    }
    if (ev) cudaEventRecord(ev[5], s);
    if (rc) return rc;
    ctx->have_step = true;
    ctx->errors_hold_m = lazy;
    ctx->steps_done += 1;
    ctx->last_stream = s;
    return PSGD_OK;
}

int psgd_step(psgd_ctx* ctx, const void* const* grads, float* const* errors, float* const* q, float* const* p_hat,
              float* const* recon, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (ctx->dist_phase != 0) return fail(ctx, PSGD_ERR_STATE, "a distributed step is in progress");
    if (ctx->L == 0) return PSGD_OK;
    const size_t WL = static_cast<size_t>(ctx->W) * ctx->L;
    int rc = check_ptr_array(ctx, grads, WL, false, "grads");
    if (!rc) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(errors), WL, false, "errors");
    if (!rc) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(q), ctx->L, false, "q");
    if (!rc && p_hat) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(p_hat), ctx->L, true, "p_hat");
    if (!rc && recon) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(recon), ctx->L, true, "recon");
    if (rc) return rc;
    DeviceGuard g(ctx->device);
    return step_impl(ctx, grads, errors, q, p_hat, recon, static_cast<cudaStream_t>(stream));
}

// Staging area of at least `need` bytes for host gradients (grown on demand).
static int ensure_stage(psgd_ctx* ctx, size_t need) {
    if (need <= ctx->stage_bytes) return PSGD_OK;
    if (ctx->stage) cudaFree(ctx->stage);
    ctx->stage = nullptr;
    ctx->stage_bytes = 0;
    cudaError_t e = cudaMalloc(&ctx->stage, need);
    if (e != cudaSuccess) return fail(ctx, PSGD_ERR_OOM, "staging of %zu bytes: %s", need, cudaGetErrorString(e));
    ctx->stage_bytes = need;
    return PSGD_OK;
}

// The step on staged gradients, then P_hat and Q_bar copied to the host.
static int step_and_download(psgd_ctx* ctx, const void* const* dev_grads, float* const* errors, float* const* q,
                             float* const* p_hat_host, float* const* q_host, cudaStream_t s,
                             const LayerGroups* groups) {
    int rc = step_impl(ctx, dev_grads, errors, q, nullptr, nullptr, s, groups);
    if (rc) return rc;
    for (int l = 0; l < ctx->L; ++l) {
        const LayerDesc& d = ctx->desc[l];
        if (p_hat_host && p_hat_host[l]) {
            // P_hat lives in the workspace with a padded row stride R
            cudaError_t e = cudaMemcpy2DAsync(p_hat_host[l], sizeof(float) * ctx->r, ctx->work.phat + d.prow_off,
                                              sizeof(float) * ctx->R, sizeof(float) * ctx->r, d.m,
                                              cudaMemcpyDeviceToHost, s);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "P_hat download");
        }
        if (q_host && q_host[l]) {
            cudaError_t e = cudaMemcpyAsync(q_host[l], q[l], sizeof(float) * d.n * ctx->r, cudaMemcpyDeviceToHost, s);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "Q download");
        }
    }
    return PSGD_OK;
}

int psgd_step_host(psgd_ctx* ctx, const void* const* grads_host, float* const* errors, float* const* q,
                   float* const* p_hat_host, float* const* q_host, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (ctx->dist_phase != 0) return fail(ctx, PSGD_ERR_STATE, "a distributed step is in progress");
    if (ctx->L == 0) return PSGD_OK;
    const size_t WL = static_cast<size_t>(ctx->W) * ctx->L;
    if (!grads_host) return fail(ctx, PSGD_ERR_ARG, "grads_host is null");
    for (size_t i = 0; i < WL; ++i)
        if (!grads_host[i]) return fail(ctx, PSGD_ERR_ARG, "grads_host[%zu] is null", i);
    int rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(errors), WL, false, "errors");
    if (!rc) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(q), ctx->L, false, "q");
    if (rc) return rc;
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t esz = ctx->dtype == PSGD_BF16 ? 2 : 4;
    // staging layout: worker-major, every matrix 256-byte aligned
    std::vector<size_t> offs(ctx->L);
    size_t per_worker = 0;
    for (int l = 0; l < ctx->L; ++l) {
        offs[l] = per_worker;
        per_worker = align_up(per_worker + static_cast<size_t>(ctx->desc[l].m * ctx->desc[l].n) * esz, 256);
    }
    rc = ensure_stage(ctx, per_worker * ctx->W);
    if (rc) return rc;
    const LayerGroups groups = upload_groups(ctx);
    rc = begin_upload(ctx, groups.size(), s);
    if (rc) return rc;
    std::vector<const void*> dev_grads(WL);
    for (size_t g = 0; g < groups.size(); ++g) {
        for (int w = 0; w < ctx->W; ++w)
            for (int l = groups[g].first; l < groups[g].second; ++l) {
                unsigned char* dst = static_cast<unsigned char*>(ctx->stage) + per_worker * w + offs[l];
                const size_t bytes = static_cast<size_t>(ctx->desc[l].m * ctx->desc[l].n) * esz;
                cudaError_t e = bytes ? cudaMemcpyAsync(dst, grads_host[w * ctx->L + l], bytes, cudaMemcpyHostToDevice,
                                                        ctx->up_stream)
                                      : cudaSuccess;
                if (e != cudaSuccess) return cuda_fail(ctx, e, "gradient upload");
                dev_grads[w * ctx->L + l] = dst;
            }
        cudaError_t e = cudaEventRecord(ctx->up_ev[g], ctx->up_stream);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "upload event");
    }
    return step_and_download(ctx, dev_grads.data(), errors, q, p_hat_host, q_host, s, &groups);
}

int psgd_step_host_flat(psgd_ctx* ctx, const void* const* grads_host, const int64_t* layer_offset,
                        float* const* errors, float* const* q, float* const* p_hat_host, float* const* q_host,
                        void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (ctx->dist_phase != 0) return fail(ctx, PSGD_ERR_STATE, "a distributed step is in progress");
    if (ctx->L == 0) return PSGD_OK;
    const size_t WL = static_cast<size_t>(ctx->W) * ctx->L;
    if (!grads_host || !layer_offset) return fail(ctx, PSGD_ERR_ARG, "grads_host or layer_offset is null");
    for (int w = 0; w < ctx->W; ++w)
        if (!grads_host[w]) return fail(ctx, PSGD_ERR_ARG, "grads_host[%d] is null", w);
    const size_t esz = ctx->dtype == PSGD_BF16 ? 2 : 4;
    size_t span = 0;   // elements per worker buffer
    for (int l = 0; l < ctx->L; ++l) {
        if (layer_offset[l] < 0) return fail(ctx, PSGD_ERR_ARG, "layer_offset[%d] < 0", l);
        if ((static_cast<size_t>(layer_offset[l]) * esz) % 16 != 0)
            return fail(ctx, PSGD_ERR_ALIGN, "layer_offset[%d] is not a multiple of 16 bytes", l);
        span = std::max(span, static_cast<size_t>(layer_offset[l] + ctx->desc[l].m * ctx->desc[l].n));
    }
    int rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(errors), WL, false, "errors");
    if (!rc) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(q), ctx->L, false, "q");
    if (rc) return rc;
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // staging layout: one 256-byte aligned slot per worker, the host layout inside
    const size_t per_worker = align_up(span * esz, 256);
    rc = ensure_stage(ctx, per_worker * ctx->W);
    if (rc) return rc;
    std::vector<const void*> dev_grads(WL);
    for (int w = 0; w < ctx->W; ++w) {
        unsigned char* dst = static_cast<unsigned char*>(ctx->stage) + per_worker * w;
        for (int l = 0; l < ctx->L; ++l) dev_grads[w * ctx->L + l] = dst + static_cast<size_t>(layer_offset[l]) * esz;
    }
    // per group: runs of layers whose element ranges follow one another in
    // the host buffer (gaps that hold no layer's elements included), one
    // copy per run and worker
    auto lend = [&](int l) { return layer_offset[l] + ctx->desc[l].m * ctx->desc[l].n; };
    auto gap_free = [&](int64_t a, int64_t b) {
        for (int k = 0; k < ctx->L; ++k)
            if (ctx->desc[k].m * ctx->desc[k].n > 0 && layer_offset[k] < b && lend(k) > a) return false;
        return true;
    };
    const LayerGroups groups = upload_groups(ctx);
    rc = begin_upload(ctx, groups.size(), s);
    if (rc) return rc;
    for (size_t g = 0; g < groups.size(); ++g) {
        for (int l = groups[g].first; l < groups[g].second;) {
            const int64_t a = layer_offset[l];
            int64_t b = lend(l);
            int k = l + 1;
            while (k < groups[g].second && layer_offset[k] >= b && gap_free(b, layer_offset[k])) b = std::max(b, lend(k++));
            if (b > a)
                for (int w = 0; w < ctx->W; ++w) {
                    const size_t off = static_cast<size_t>(a) * esz;
                    cudaError_t e = cudaMemcpyAsync(static_cast<unsigned char*>(ctx->stage) + per_worker * w + off,
                                                    static_cast<const unsigned char*>(grads_host[w]) + off,
                                                    static_cast<size_t>(b - a) * esz, cudaMemcpyHostToDevice,
                                                    ctx->up_stream);
                    if (e != cudaSuccess) return cuda_fail(ctx, e, "gradient upload");
                }
            l = k;
        }
        cudaError_t e = cudaEventRecord(ctx->up_ev[g], ctx->up_stream);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "upload event");
    }
    return step_and_download(ctx, dev_grads.data(), errors, q, p_hat_host, q_host, s, &groups);
}

int psgd_materialize_errors(psgd_ctx* ctx, float* const* errors, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (!(ctx->flags & PSGD_FLAG_LAZY_ERRORS)) return fail(ctx, PSGD_ERR_STATE, "context is not in lazy-error mode");
    if (ctx->L == 0 || !ctx->errors_hold_m) return PSGD_OK;
    const size_t WL = static_cast<size_t>(ctx->W) * ctx->L;
    int rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(errors), WL, false, "errors");
    if (rc) return rc;
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::vector<uint64_t> te(WL);
    for (size_t i = 0; i < WL; ++i) te[i] = reinterpret_cast<uint64_t>(errors[i]);
    cudaError_t e = ctx->tab_e.update(te, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "table upload");
    psgd::Params p = base_params(ctx);
    p.t.errors = static_cast<float* const*>(ctx->tab_e.dev());
    p.do_resid = 1;
    rc = launch(ctx, 2, true, p, ctx->smem_c, s);
    if (rc) return rc;
    ctx->errors_hold_m = false;
    ctx->last_stream = s;
    return PSGD_OK;
}

int psgd_momentum_step(psgd_ctx* ctx, float* const* params, float* const* mom, float lr, float beta, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (ctx->L == 0) return PSGD_OK;
    if (!ctx->have_step) return fail(ctx, PSGD_ERR_STATE, "no step has run yet");
    int rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(params), ctx->L, false, "params");
    if (!rc) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(mom), ctx->L, false, "mom");
    if (rc) return rc;
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::vector<uint64_t> tm(2 * ctx->L);
    for (int l = 0; l < ctx->L; ++l) {
        tm[l] = reinterpret_cast<uint64_t>(params[l]);
        tm[ctx->L + l] = reinterpret_cast<uint64_t>(mom[l]);
    }
    cudaError_t e = ctx->tab_m.update(tm, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "table upload");
    psgd::Params p = base_params(ctx);
    void* const* mt = static_cast<void* const*>(ctx->tab_m.dev());
    p.t.params = reinterpret_cast<float* const*>(mt);
    p.t.mom = reinterpret_cast<float* const*>(mt + ctx->L);
    p.do_mom = 1;
    p.lr = lr;
    p.beta = beta;
    rc = launch(ctx, 2, (ctx->flags & PSGD_FLAG_LAZY_ERRORS) != 0, p, ctx->smem_c, s);
    if (rc) return rc;
    ctx->last_stream = s;
    return PSGD_OK;
}

int psgd_vec_mean(psgd_ctx* ctx, const float* const* vecs, float* const* out, const int64_t* len, int count,
                  float* const* params, float* const* mom, float lr, float beta, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (count < 0) return fail(ctx, PSGD_ERR_ARG, "count < 0");
    if (count == 0) return PSGD_OK;
    if (!len) return fail(ctx, PSGD_ERR_ARG, "len is null");
    if (count > 65535) return fail(ctx, PSGD_ERR_ARG, "too many vectors");
    if ((params == nullptr) != (mom == nullptr)) return fail(ctx, PSGD_ERR_ARG, "params and mom go together");
    const size_t WK = static_cast<size_t>(ctx->W) * count;
    if (!vecs || !out) return fail(ctx, PSGD_ERR_ARG, "null pointer array");
    int64_t maxlen = 0;
    for (int k = 0; k < count; ++k) {
        if (len[k] < 0) return fail(ctx, PSGD_ERR_ARG, "len[%d] < 0", k);
        maxlen = std::max(maxlen, len[k]);
        // an empty vector's pointers are never dereferenced (and may be null)
        if (len[k] == 0) continue;
        const void* ps[3] = {out[k], params ? params[k] : nullptr, mom ? mom[k] : nullptr};
        for (int j = 0; j < 3; ++j) {
            if (j > 0 && !params) break;
            if (!ps[j]) return fail(ctx, PSGD_ERR_ARG, "null pointer for vector %d", k);
            if (!aligned16(ps[j])) return fail(ctx, PSGD_ERR_ALIGN, "vector %d: pointer not 16-byte aligned", k);
        }
        for (int w = 0; w < ctx->W; ++w) {
            const void* v = vecs[static_cast<size_t>(w) * count + k];
            if (!v) return fail(ctx, PSGD_ERR_ARG, "vecs[%d][%d] is null", w, k);
            if (!aligned16(v)) return fail(ctx, PSGD_ERR_ALIGN, "vecs[%d][%d] is not 16-byte aligned", w, k);
        }
    }
    if (maxlen == 0) return PSGD_OK;
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // table: vecs[W*K] | out[K] | params[K] | mom[K] | len[K]
    std::vector<uint64_t> tv(WK + 4 * static_cast<size_t>(count), 0);
    for (size_t i = 0; i < WK; ++i) tv[i] = reinterpret_cast<uint64_t>(vecs[i]);
    for (int k = 0; k < count; ++k) {
        tv[WK + k] = reinterpret_cast<uint64_t>(out[k]);
        tv[WK + count + k] = params ? reinterpret_cast<uint64_t>(params[k]) : 0;
        tv[WK + 2 * count + k] = mom ? reinterpret_cast<uint64_t>(mom[k]) : 0;
        tv[WK + 3 * count + k] = static_cast<uint64_t>(len[k]);
    }
    cudaError_t e = ctx->tab_v.update(tv, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "table upload");
    uint64_t* t = static_cast<uint64_t*>(ctx->tab_v.dev());
    const unsigned gx = static_cast<unsigned>(std::min<int64_t>(256, (maxlen + 255) / 256));
    psgd::k_vec_mean<<<dim3(gx, count), 256, 0, s>>>(
        reinterpret_cast<const float* const*>(t), reinterpret_cast<float* const*>(t + WK),
        reinterpret_cast<const int64_t*>(t + WK + 3 * count), count, ctx->W,
        1.0f / static_cast<float>(ctx->w_global > 0 ? ctx->w_global : ctx->W),
        params ? reinterpret_cast<float* const*>(t + WK + count) : nullptr,
        mom ? reinterpret_cast<float* const*>(t + WK + 2 * count) : nullptr, lr, beta);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "vec_mean launch");
    ctx->last_stream = s;
    return PSGD_OK;
}

// ---- allocation-free single-layer step ------------------------------------
// All scratch of psgd_step_static lives in this array; host code never uses
// its name as an address: the device address comes from
// cudaGetSymbolAddress, looked up once per device.  The first 256 bytes
// hold the status word of the last call (kStaticStatusOffset); the layer's
// scratch follows.
static __device__ __align__(256) unsigned char g_psgd_static_scratch[PSGD_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kStaticStatusOffset = 0;
constexpr size_t kStaticHeader = 256;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};
// dynamic shared memory each kernel was opted in to on each device by this
// entry point: [device][pass][log2 R][dtype] (bytes, 0 = not yet)
size_t g_static_smem[kMaxDevices][3][6][2] = {};

int log2_rank(int R) {
    int k = 0;
    while ((1 << k) < R) ++k;
    return k;
}

cudaError_t static_scratch_address(void** out, int* dev_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_psgd_static_scratch);
        if (e != cudaSuccess) return e;
        g_static_addr[dev] = p;
    }
    *out = g_static_addr[dev];
    *dev_out = dev;
    return cudaSuccess;
}

// Raise a kernel's dynamic shared-memory limit once per (device, kernel,
// size): later calls only read the cache.
cudaError_t static_smem_opt_in(int dev, int which, int R, int dtype, const void* fn, size_t need) {
    std::lock_guard<std::mutex> lock(g_static_mu);
    size_t& have = g_static_smem[dev][which][log2_rank(R)][dtype == PSGD_BF16 ? 1 : 0];
    if (have >= need) return cudaSuccess;
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return e;
    if (static_cast<size_t>(fa.maxDynamicSharedSizeBytes) < need) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(need));
        if (e != cudaSuccess) return e;
    }
    have = need;
    return cudaSuccess;
}

// Everything a call writes into the scratch before its three passes,
// passed by value (no host staging buffer): the layer descriptor, the
// pointer table (grads[W], errors[W], q, p_hat, recon) and the extents to
// clear (tile map, counters) plus the status word.
struct StaticSetup {
    LayerDesc desc;
    uint64_t tab[2 * psgd::kMaxWorkers + 3];
    LayerDesc* desc_dst;
    uint64_t* tab_dst;
    int* tile_dst;
    unsigned* cnt_dst;
    int* status_dst;
    int ntab;
    int64_t ntiles, ncnt;
};

__global__ void k_static_setup(const StaticSetup s) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    if (tid == 0) {
        *s.desc_dst = s.desc;
        *s.status_dst = 0;
    }
    for (int64_t i = tid; i < s.ntab; i += stride) s.tab_dst[i] = s.tab[i];
    // one layer: every tile maps to layer 0; counters start at zero
    for (int64_t i = tid; i < s.ntiles; i += stride) s.tile_dst[i] = 0;
    for (int64_t i = tid; i < s.ncnt; i += stride) s.cnt_dst[i] = 0u;
}

}  // namespace

int psgd_step_static(int64_t m, int64_t n, int rank, int workers, int grad_dtype, const void* const* grads,
                     float* const* errors, float* q, float* p_hat, float* recon, void* stream) {
    g_create_error.clear();
    if (rank < 1 || rank > psgd::kMaxRank) return fail(nullptr, PSGD_ERR_ARG, "rank %d not in [1, 32]", rank);
    if (workers < 1 || workers > psgd::kMaxWorkers)
        return fail(nullptr, PSGD_ERR_ARG, "workers %d not in [1, %d]", workers, psgd::kMaxWorkers);
    if (grad_dtype != PSGD_F32 && grad_dtype != PSGD_BF16) return fail(nullptr, PSGD_ERR_ARG, "bad grad dtype");
    if (m < 1 || n < 1 || rank > m || rank > n || m > (int64_t(1) << 31) || n > (int64_t(1) << 31))
        return fail(nullptr, PSGD_ERR_ARG, "bad shape %lld x %lld for rank %d", (long long)m, (long long)n, rank);
    if (!grads || !errors || !q) return fail(nullptr, PSGD_ERR_ARG, "null pointer argument");
    for (int w = 0; w < workers; ++w) {
        if (!grads[w] || !errors[w]) return fail(nullptr, PSGD_ERR_ARG, "null pointer for worker %d", w);
        if (!aligned16(grads[w]) || !aligned16(errors[w]))
            return fail(nullptr, PSGD_ERR_ALIGN, "pointer of worker %d is not 16-byte aligned", w);
    }
    if (!aligned16(q) || (p_hat && !aligned16(p_hat)) || (recon && !aligned16(recon)))
        return fail(nullptr, PSGD_ERR_ALIGN, "q, p_hat or recon is not 16-byte aligned");

    // tile geometry of the one layer (same rules as a context's)
    const int R = pad_rank(rank);
    LayerSizes sz{};
    LayerDesc d = layer_geometry(m, n, R, workers, &sz);
    const int64_t ntiles = sz.tiles;

    // scratch layout inside the static array (after the status header)
    size_t off = kStaticHeader;
    auto carve = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + std::max<size_t>(bytes, 1), 256);
        return o;
    };
    const int ntab = 2 * workers + 3;
    const size_t o_desc = carve(sizeof(LayerDesc));
    const size_t o_tab = carve(sizeof(uint64_t) * ntab);
    const size_t o_tile = carve(sizeof(int) * ntiles);
    const size_t o_pbar = carve(sizeof(double) * sz.prow);
    const size_t o_phat = carve(sizeof(float) * sz.prow);
    const size_t o_qbar = carve(sizeof(float) * sz.qrow);
    const size_t o_ppart = carve(sizeof(double) * sz.ppart);
    const size_t o_qpart = carve(sizeof(double) * sz.qpart);
    const size_t o_gram = carve(sizeof(double) * sz.gram);
    const size_t o_gsup = carve(sizeof(double) * sz.gsup);
    const size_t o_qsup = carve(sizeof(double) * sz.qsup);
    const size_t o_T = carve(sizeof(double) * sz.t);
    const size_t o_cnt = carve(sizeof(unsigned) * sz.cnt);
    if (off > PSGD_STATIC_SCRATCH_BYTES)
        return fail(nullptr, PSGD_ERR_ARG, "layer %lld x %lld at rank %d with %d workers needs %zu bytes of scratch; "
                    "the static scratch holds %u", (long long)m, (long long)n, rank, workers, off,
                    PSGD_STATIC_SCRATCH_BYTES);
    // every array of the one layer starts at its own piece: offsets are 0
    d.tile_begin = 0;
    d.prow_off = d.qrow_off = d.ppart_off = d.qpart_off = d.gram_off = d.gsup_off = d.qsup_off = d.t_off =
        d.cnt_off = 0;

    void* base_v = nullptr;
    int dev = 0;
    cudaError_t e = static_scratch_address(&base_v, &dev);
    if (e != cudaSuccess) return fail(nullptr, PSGD_ERR_CUDA, "static scratch address: %s", cudaGetErrorString(e));
    unsigned char* base = static_cast<unsigned char*>(base_v);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    const size_t smem[3] = {smem_need(0, R, workers, d.tm, d.vec), smem_need(1, R, workers, d.tm, d.vec),
                            smem_need(2, R, workers, d.tm, d.vec)};
    void* fns[3];
    for (int which = 0; which < 3; ++which) {
        fns[which] = kernel_ptr(which, R, grad_dtype, false, false);
        e = static_smem_opt_in(dev, which, R, grad_dtype, fns[which], smem[which]);
        if (e != cudaSuccess) return fail(nullptr, PSGD_ERR_CUDA, "shared-memory opt-in: %s", cudaGetErrorString(e));
    }

    // descriptor, pointer table, tile map, counters and status written on
    // the device by one set-up kernel that takes them by value
    StaticSetup su{};
    su.desc = d;
    for (int w = 0; w < workers; ++w) {
        su.tab[w] = reinterpret_cast<uint64_t>(grads[w]);
        su.tab[workers + w] = reinterpret_cast<uint64_t>(errors[w]);
    }
    su.tab[2 * workers] = reinterpret_cast<uint64_t>(q);
    su.tab[2 * workers + 1] = reinterpret_cast<uint64_t>(p_hat);
    su.tab[2 * workers + 2] = reinterpret_cast<uint64_t>(recon);
    su.desc_dst = reinterpret_cast<LayerDesc*>(base + o_desc);
    su.tab_dst = reinterpret_cast<uint64_t*>(base + o_tab);
    su.tile_dst = reinterpret_cast<int*>(base + o_tile);
    su.cnt_dst = reinterpret_cast<unsigned*>(base + o_cnt);
    su.status_dst = reinterpret_cast<int*>(base + kStaticStatusOffset);
    su.ntab = ntab;
    su.ntiles = ntiles;
    su.ncnt = sz.cnt;
    {
        const int64_t work = std::max<int64_t>({ntiles, sz.cnt, static_cast<int64_t>(ntab), 1});
        const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(148, (work + 255) / 256));
        k_static_setup<<<blocks, 256, 0, s>>>(su);
        e = cudaGetLastError();
        if (e != cudaSuccess) return fail(nullptr, PSGD_ERR_CUDA, "scratch set-up: %s", cudaGetErrorString(e));
    }

    psgd::Params p{};
    uint64_t* tab_d = reinterpret_cast<uint64_t*>(base + o_tab);
    p.t.layers = reinterpret_cast<const LayerDesc*>(base + o_desc);
    p.t.tile_layer = reinterpret_cast<const int*>(base + o_tile);
    p.t.grads = reinterpret_cast<const void* const*>(tab_d);
    p.t.errors = reinterpret_cast<float* const*>(tab_d + workers);
    p.t.q = reinterpret_cast<float* const*>(tab_d + 2 * workers);
    p.t.p_hat_out = reinterpret_cast<float* const*>(tab_d + 2 * workers + 1);
    p.t.recon_out = reinterpret_cast<float* const*>(tab_d + 2 * workers + 2);
    p.ws.pbar = reinterpret_cast<double*>(base + o_pbar);
    p.ws.phat = reinterpret_cast<float*>(base + o_phat);
    p.ws.qbar = reinterpret_cast<float*>(base + o_qbar);
    p.ws.ppart = reinterpret_cast<double*>(base + o_ppart);
    p.ws.qpart = reinterpret_cast<double*>(base + o_qpart);
    p.ws.gram = reinterpret_cast<double*>(base + o_gram);
    p.ws.gsup = reinterpret_cast<double*>(base + o_gsup);
    p.ws.qsup = reinterpret_cast<double*>(base + o_qsup);
    p.ws.T = reinterpret_cast<double*>(base + o_T);
    p.ws.cnt = reinterpret_cast<unsigned*>(base + o_cnt);
    p.ws.status = reinterpret_cast<int*>(base + kStaticStatusOffset);
    p.num_layers = 1;
    p.workers = workers;
    p.r = rank;
    p.inv_w = 1.0f / static_cast<float>(workers);
    p.drop_tol = kDropTol;
    p.inv_w_global = 1.0 / static_cast<double>(workers);

    for (int which = 0; which < 3; ++which) {
        psgd::Params pw = p;
        if (which == 2) {
            pw.do_resid = 1;
            pw.do_recon = recon ? 1 : 0;
        }
        void* args[] = {&pw};
        if (which == 1) {
            e = cudaLaunchKernel(kernel_ptr(7, R, grad_dtype, false, false), phat_grid(d.m, 1, R),
                                 dim3(psgd::kThreads), args, 0, s);
            if (e != cudaSuccess) return fail(nullptr, PSGD_ERR_CUDA, "P_hat launch: %s", cudaGetErrorString(e));
        }
        e = cudaLaunchKernel(fns[which], dim3(static_cast<unsigned>(ntiles)), dim3(psgd::kThreads), args,
                             smem[which], s);
        if (e != cudaSuccess) return fail(nullptr, PSGD_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
    }
    return PSGD_OK;
}

int psgd_step_static_status(void* stream) {
    g_create_error.clear();
    void* base_v = nullptr;
    int dev = 0;
    cudaError_t e = static_scratch_address(&base_v, &dev);
    if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    int word = 0;
    if (e == cudaSuccess)
        e = cudaMemcpy(&word, static_cast<unsigned char*>(base_v) + kStaticStatusOffset, sizeof(int),
                       cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(nullptr, PSGD_ERR_CUDA, "static status: %s", cudaGetErrorString(e));
    if (word & psgd::kStatusTimeout)
        return fail(nullptr, PSGD_ERR_TIMEOUT, "device status word 0x%x: a bounded wait ran out", word);
    if (word != 0)
        return fail(nullptr, PSGD_ERR_DEVICE, "device status word 0x%x: a reduction counter was inconsistent "
                    "(calls overlapping on the GPU)", word);
    return PSGD_OK;
}

// ---- distributed step (the all-reduces between the calls are the caller's)

int psgd_set_global_workers(psgd_ctx* ctx, int total) {
    if (!ctx) return PSGD_ERR_ARG;
    if (total < ctx->W) return fail(ctx, PSGD_ERR_ARG, "global workers %d < local workers %d", total, ctx->W);
    ctx->w_global = total;
    return PSGD_OK;
}

int psgd_dist_sizes(const psgd_ctx* ctx, size_t* p_elems, size_t* q_elems) {
    if (!ctx || !p_elems || !q_elems) return PSGD_ERR_ARG;
    size_t pe = 0, qe = 0;
    for (auto& d : ctx->desc) {
        pe += static_cast<size_t>(d.m) * ctx->R;
        qe += static_cast<size_t>(d.n) * ctx->R;
    }
    *p_elems = pe;
    *q_elems = qe;
    return PSGD_OK;
}

static psgd::Params dist_params(psgd_ctx* ctx) {
    psgd::Params p = base_params(ctx);
    const size_t WL = static_cast<size_t>(ctx->W) * ctx->L;
    void* const* wt = static_cast<void* const*>(ctx->tab_w.dev());
    void* const* lt = static_cast<void* const*>(ctx->tab_l.dev());
    p.t.grads = reinterpret_cast<const void* const*>(wt);
    p.t.errors = reinterpret_cast<float* const*>(wt + WL);
    p.t.q = reinterpret_cast<float* const*>(lt);
    p.t.p_hat_out = reinterpret_cast<float* const*>(lt + ctx->L);
    p.t.recon_out = reinterpret_cast<float* const*>(lt + 2 * ctx->L);
    p.dist = 1;
    return p;
}

int psgd_dist_p(psgd_ctx* ctx, const void* const* grads, float* const* errors, float* const* q, float* const* p_hat,
                float* const* recon, double* p_send, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (ctx->dist_phase != 0) return fail(ctx, PSGD_ERR_STATE, "psgd_dist_p called in the middle of a step");
    if (ctx->iters != 1 || ctx->svd_every > 0)
        return fail(ctx, PSGD_ERR_STATE, "the distributed step does one power iteration without SVD refresh");
    if (ctx->L == 0) return PSGD_OK;
    const size_t WL = static_cast<size_t>(ctx->W) * ctx->L;
    int rc = check_ptr_array(ctx, grads, WL, false, "grads");
    if (!rc) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(errors), WL, false, "errors");
    if (!rc) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(q), ctx->L, false, "q");
    if (!rc && p_hat) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(p_hat), ctx->L, true, "p_hat");
    if (!rc && recon) rc = check_ptr_array(ctx, reinterpret_cast<const void* const*>(recon), ctx->L, true, "recon");
    if (!rc && (!p_send || !aligned16(p_send))) rc = fail(ctx, PSGD_ERR_ALIGN, "p_send null or not 16-byte aligned");
    if (rc) return rc;
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::vector<uint64_t> tw(2 * WL);
    for (size_t i = 0; i < WL; ++i) {
        tw[i] = reinterpret_cast<uint64_t>(grads[i]);
        tw[WL + i] = reinterpret_cast<uint64_t>(errors[i]);
    }
    std::vector<uint64_t> tl(3 * ctx->L, 0);
    for (int l = 0; l < ctx->L; ++l) {
        tl[l] = reinterpret_cast<uint64_t>(q[l]);
        tl[ctx->L + l] = p_hat ? reinterpret_cast<uint64_t>(p_hat[l]) : 0;
        tl[2 * ctx->L + l] = recon ? reinterpret_cast<uint64_t>(recon[l]) : 0;
    }
    cudaError_t e = ctx->tab_w.update(tw, s);
    if (e == cudaSuccess) e = ctx->tab_l.update(tl, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "table upload");
    const bool lazy = (ctx->flags & PSGD_FLAG_LAZY_ERRORS) != 0;
    psgd::Params p = dist_params(ctx);
    p.use_prev = (lazy && ctx->errors_hold_m) ? 1 : 0;
    p.dist_out = p_send;
    if (ctx->flags & PSGD_FLAG_NO_WARM_START) {
        int64_t maxn = 0;
        for (auto& d : ctx->desc) maxn = std::max(maxn, d.n);
        const int64_t blocks4 = (maxn * ctx->r + 3) / 4;
        const unsigned gx = static_cast<unsigned>(std::min<int64_t>(1024, (blocks4 + 255) / 256));
        psgd::k_init_q<<<dim3(std::max(1u, gx), ctx->L), 256, 0, s>>>(p.t.q, ctx->desc_d, ctx->r, ctx->seed,
                                                                      ctx->steps_done + 1);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(ctx, e, "fresh Q launch");
    }
    cudaEvent_t* ev = profile_events(ctx, &e);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "profiling event");
    ctx->dist_ev = ev;
    if (ev) cudaEventRecord(ev[0], s);
    rc = launch(ctx, 0, lazy, p, ctx->smem_a, s);
    if (ev) cudaEventRecord(ev[1], s);
    if (rc) return rc;
    ctx->tab_l_has_recon = recon != nullptr;
    ctx->dist_phase = 1;
    ctx->last_stream = s;
    return PSGD_OK;
}

int psgd_dist_q(psgd_ctx* ctx, const double* p_sum, double* q_send, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (ctx->L == 0) return PSGD_OK;
    if (ctx->dist_phase != 1) return fail(ctx, PSGD_ERR_STATE, "psgd_dist_q must follow psgd_dist_p");
    if (!p_sum || !q_send || !aligned16(p_sum) || !aligned16(q_send))
        return fail(ctx, PSGD_ERR_ALIGN, "p_sum / q_send null or not 16-byte aligned");
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool lazy = (ctx->flags & PSGD_FLAG_LAZY_ERRORS) != 0;
    psgd::Params p = dist_params(ctx);
    p.dist_in = p_sum;
    void* fn = kernel_ptr(5, ctx->R, ctx->dtype, false, false);
    void* args[] = {&p};
    cudaEvent_t* ev = ctx->dist_ev;
    if (ev) cudaEventRecord(ev[2], s);
    cudaError_t e = cudaLaunchKernel(fn, dim3(static_cast<unsigned>(ctx->L)), dim3(psgd::kThreads), args, 0, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "distributed orthogonalisation launch");
    p.dist_in = nullptr;
    p.dist_out = q_send;
    int rc = launch(ctx, 1, lazy, p, ctx->smem_b, s);
    if (ev) cudaEventRecord(ev[3], s);
    if (rc) return rc;
    ctx->dist_phase = 2;
    return PSGD_OK;
}

int psgd_dist_finish(psgd_ctx* ctx, const double* q_sum, void* stream) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->err.clear();
    if (ctx->L == 0) return PSGD_OK;
    if (ctx->dist_phase != 2) return fail(ctx, PSGD_ERR_STATE, "psgd_dist_finish must follow psgd_dist_q");
    if (!q_sum || !aligned16(q_sum)) return fail(ctx, PSGD_ERR_ALIGN, "q_sum null or not 16-byte aligned");
    DeviceGuard g(ctx->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool lazy = (ctx->flags & PSGD_FLAG_LAZY_ERRORS) != 0;
    psgd::Params p = dist_params(ctx);
    p.dist = 0;
    p.dist_in = q_sum;
    int64_t maxn = 0;
    for (auto& d : ctx->desc) maxn = std::max(maxn, d.n);
    const unsigned gx = static_cast<unsigned>(std::min<int64_t>(1024, (maxn * ctx->R + 255) / 256));
    void* fn = kernel_ptr(6, ctx->R, ctx->dtype, false, false);
    void* args[] = {&p};
    cudaEvent_t* ev = ctx->dist_ev;
    if (ev) cudaEventRecord(ev[4], s);
    cudaError_t e = cudaLaunchKernel(fn, dim3(std::max(1u, gx), static_cast<unsigned>(ctx->L)), dim3(256), args, 0, s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "distributed Q_bar launch");
    const bool recon = ctx->tab_l_has_recon;
    if (!lazy || recon) {
        psgd::Params pc = p;
        pc.dist_in = nullptr;
        pc.do_resid = lazy ? 0 : 1;
        pc.do_recon = recon ? 1 : 0;
        int rc = launch(ctx, 2, lazy, pc, ctx->smem_c, s);
        if (rc) return rc;
    }
    if (ev) cudaEventRecord(ev[5], s);
    ctx->dist_ev = nullptr;
    ctx->dist_phase = 0;
    ctx->have_step = true;
    ctx->errors_hold_m = lazy;
    ctx->steps_done += 1;
    return PSGD_OK;
}

int psgd_set_power_iters(psgd_ctx* ctx, int iters) {
    if (!ctx) return PSGD_ERR_ARG;
    if (iters < 1 || iters > 8) return fail(ctx, PSGD_ERR_ARG, "power iterations %d not in [1, 8]", iters);
    ctx->iters = iters;
    return PSGD_OK;
}

// (Re)build the rank r + p context of oversampled refresh steps, or drop it
// when refresh is off or no column can be added (r + p capped by 32 and by
// the smallest side of every layer).
static int configure_refresh(psgd_ctx* ctx) {
    int rp = std::min(psgd::kMaxRank, ctx->r + ctx->svd_over);
    for (auto& sh : ctx->shapes) rp = static_cast<int>(std::min<int64_t>(rp, std::min(sh.m, sh.n)));
    const bool want = ctx->svd_every > 0 && rp > ctx->r && ctx->L > 0;
    if (ctx->sub && (!want || ctx->sub->r != rp)) {
        psgd_destroy(ctx->sub);
        ctx->sub = nullptr;
        if (ctx->qsub) cudaFree(ctx->qsub);
        ctx->qsub = nullptr;
        ctx->tab_sub.release();
        ctx->tab_sub_vals.clear();
    }
    if (!want || ctx->sub) return PSGD_OK;
    DeviceGuard g(ctx->device);
    psgd_ctx* sub = nullptr;
    int rc = psgd_create(&sub, ctx->shapes.data(), ctx->L, rp, ctx->W, ctx->seed, ctx->dtype,
                         ctx->flags & PSGD_FLAG_SUM_FIRST);
    if (rc) return fail(ctx, rc, "refresh context: %s", psgd_last_error(nullptr));
    std::vector<size_t> offs(ctx->L);
    size_t total = 0;
    for (int l = 0; l < ctx->L; ++l) {
        offs[l] = total;
        total = align_up(total + static_cast<size_t>(ctx->shapes[l].n) * rp * sizeof(float), 256);
    }
    cudaError_t e = cudaMalloc(&ctx->qsub, total);
    if (e != cudaSuccess) {
        psgd_destroy(sub);
        return fail(ctx, PSGD_ERR_OOM, "refresh Q block of %zu bytes: %s", total, cudaGetErrorString(e));
    }
    ctx->sub = sub;
    ctx->tab_sub_vals.assign(3 * static_cast<size_t>(ctx->L), 0);
    for (int l = 0; l < ctx->L; ++l)
        ctx->tab_sub_vals[l] = reinterpret_cast<uint64_t>(static_cast<unsigned char*>(static_cast<void*>(ctx->qsub)) +
                                                          offs[l]);
    return PSGD_OK;
}

int psgd_set_svd_refresh(psgd_ctx* ctx, int every, int iters) {
    if (!ctx) return PSGD_ERR_ARG;
    if (every < 0) return fail(ctx, PSGD_ERR_ARG, "refresh period %d < 0", every);
    if (every > 0 && (iters < 1 || iters > 64))
        return fail(ctx, PSGD_ERR_ARG, "refresh iterations %d not in [1, 64]", iters);
    ctx->svd_every = every;
    ctx->svd_iters = every > 0 ? iters : 0;
    return configure_refresh(ctx);
}

int psgd_set_svd_oversampling(psgd_ctx* ctx, int extra) {
    if (!ctx) return PSGD_ERR_ARG;
    if (extra < 0 || extra > psgd::kMaxRank - 1)
        return fail(ctx, PSGD_ERR_ARG, "oversampling %d not in [0, %d]", extra, psgd::kMaxRank - 1);
    ctx->svd_over = extra;
    return configure_refresh(ctx);
}

int psgd_test_stall_products(psgd_ctx* ctx, int on) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->stall_products = on != 0;
    return PSGD_OK;
}

int psgd_profile_enable(psgd_ctx* ctx, int enable) {
    if (!ctx) return PSGD_ERR_ARG;
    ctx->profiling = enable != 0;
    return PSGD_OK;
}

int psgd_profile_read(psgd_ctx* ctx, double* ms, int* steps) {
    if (!ctx || !ms || !steps) return PSGD_ERR_ARG;
    DeviceGuard g(ctx->device);
    ms[0] = ms[1] = ms[2] = 0.0;
    for (size_t i = 0; i < ctx->prof_used; ++i) {
        auto& a = ctx->prof_ev[i];
        cudaError_t e = cudaEventSynchronize(a[5]);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "profile sync");
        for (int k = 0; k < 3; ++k) {
            float t = 0.f;
            e = cudaEventElapsedTime(&t, a[2 * k], a[2 * k + 1]);
            if (e != cudaSuccess) return cuda_fail(ctx, e, "profile elapsed");
            ms[k] += t;
        }
    }
    *steps = static_cast<int>(ctx->prof_used);
    ctx->prof_used = 0;
    return PSGD_OK;
}

int psgd_status(psgd_ctx* ctx) {
    if (!ctx) return PSGD_ERR_ARG;
    DeviceGuard g(ctx->device);
    cudaError_t e = cudaStreamSynchronize(ctx->last_stream);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "synchronise");
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(ctx, e, "pending error");
    int st = 0;
    e = cudaMemcpy(&st, ctx->work.status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "status read");
    if (st) {
        // reported once: the word is cleared for the steps that follow
        e = cudaMemset(ctx->work.status, 0, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(ctx, e, "status clear");
        if (st & psgd::kStatusTimeout)
            return fail(ctx, PSGD_ERR_TIMEOUT, "device status word 0x%x: a bounded wait ran out", st);
        return fail(ctx, PSGD_ERR_DEVICE, "device status word 0x%x: a reduction counter was inconsistent", st);
    }
    return PSGD_OK;
}

}  // extern "C"
