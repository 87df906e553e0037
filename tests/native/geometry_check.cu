// Host-side check of the library's own tile geometry and shared-memory
// sizing (csrc/psgd.cu included as is) over the shapes, ranks and worker
// counts the GPU tests use; run on the CPU, no device call is made.
#include "psgd.cu"
#include <cstdio>
int main() {
    struct Case { int64_t m, n; int r, W; };
    std::vector<Case> cs;
    int64_t mixed[][2] = {{300,650},{64,576},{40,130},{256,128},{33,37},{700,33},{129,1000}};
    for (int r : {1,2,3,4,8,16,32}) for (int W : {1,3,16,64,256}) for (auto& s : mixed) cs.push_back({s[0], s[1], r, W});
    int64_t full[][3] = {{2,64,2},{50,2,2},{4,90,4},{70,4,4},{8,100,8},{100,8,8},{16,160,16},{200,16,16},{32,400,32},{300,32,32},
                         {96,130,16},{40,64,16},{1,64,1},{9,7,1},{35,33,8},{1,40,1},{8,8,1}};
    for (auto& f : full) for (int W : {1,2,3,256}) cs.push_back({f[0], f[1], (int)f[2], W});
    // the full-size workloads: ResNet-18 set (r = 2, W = 16), LSTM set (r = 4,
    // W = 16), transformer set (r = 4, W = 4), the two sweeps (W = 8, r = 1..32)
    int64_t resnet[][2] = {{64,576},{128,576},{128,1152},{256,1152},{256,2304},{512,2304},{512,4608},
                           {128,64},{256,128},{512,256},{10,512}};
    for (auto& s : resnet) cs.push_back({s[0], s[1], 2, 16});
    cs.push_back({2600, 650, 4, 16});
    cs.push_back({33280, 650, 4, 16});
    int64_t tf[][2] = {{4096,12288},{4096,4096},{16384,4096},{4096,16384}};
    const auto& tf4 = tf;
    // the ResNet-18 set's 20 matrices in list order
    const int64_t resnet20[][2] = {{64,576},{64,576},{64,576},{64,576},{128,576},{128,1152},{128,1152},{128,1152},
                                   {256,1152},{256,2304},{256,2304},{256,2304},{512,2304},{512,4608},{512,4608},
                                   {512,4608},{128,64},{256,128},{512,256},{10,512}};
    for (auto& s : tf) cs.push_back({s[0], s[1], 4, 4});
    for (int r : {1,2,3,4,8,16,32}) {
        cs.push_back({8192, 8192, r, 8});
        cs.push_back({1024, 1024, r, 8});
    }
    int bad = 0, n = 0;
    for (auto& c : cs) {
        if (c.r > c.m || c.r > c.n) continue;
        const int R = pad_rank(c.r);
        LayerSizes sz{};
        LayerDesc d = layer_geometry(c.m, c.n, R, c.W, &sz);
        ++n;
        auto fail = [&](const char* what) { ++bad; std::printf("FAIL %s: m=%lld n=%lld r=%d W=%d tm=%d vec=%d slots=%d nchunk=%d\n", what,
            (long long)c.m, (long long)c.n, c.r, c.W, d.tm, d.vec, d.slots, d.nchunk); };
        if (c.n % d.vec) fail("vec divides n");
        if (d.vec > max_vec_for_rank(R)) fail("vec within the rank's limit");
        if (d.slots < 1 || d.slots > 32) fail("slots in 1..32");
        if ((int64_t)d.nchunk * d.slots < d.nvec || (int64_t)(d.nchunk - 1) * d.slots >= d.nvec) fail("chunks cover the row, none empty");
        if ((int64_t)d.nrb * d.tm < c.m || (int64_t)(d.nrb - 1) * d.tm >= c.m) fail("row blocks cover the matrix, none empty");
        if (d.tm % 8) fail("tm multiple of 8");
        if (R >= 16 && d.tm != 16 && d.tm != 32 && d.tm != 64) fail("tensor-core tiles of 16/32/64 rows");
        if ((int64_t)d.tm * R > kRowsFloatsMax) fail("rows buffer");
        if (d.slots * d.vec > 4 * psgd::kWideCols) fail("chunk within the k-steps");
        for (int lazy = 0; lazy < 2; ++lazy) {
            size_t a = smem_need(0, R, c.W, d.tm, d.vec, lazy), b = smem_need(1, R, c.W, d.tm, d.vec), cc = smem_need(2, R, c.W, d.tm, d.vec);
            if (a > 232448 || b > 232448 || cc > 232448 || !a || !b || !cc) fail("shared memory within 227 KB");
            // the CTAs per SM the launch bounds aim at (228 KB per SM, 1 KB
            // reserved per CTA): 3 for passes A and B at R <= 8, else 2
            const size_t per3 = 228 * 1024 / 3 - 1024, per2 = 228 * 1024 / 2 - 1024;
            if (a > (R <= 8 ? per3 : per2) || b > (R <= 8 ? per3 : per2) || cc > per2)
                fail("shared memory lets the intended CTAs per SM reside");
            // pass B on the 5th-generation tensor cores (R >= 16, 16-byte
            // rows): the CTAs that shared memory lets reside on one SM never
            // ask for more than its 512 TMEM columns, so no allocation waits
            if (R >= 16 && d.vec == 4) {
                const size_t resident = 228 * 1024 / (b + 1024);
                const uint32_t cols = R == 16 ? psgd::TcSmem<16>::tmem_cols : psgd::TcSmem<32>::tmem_cols;
                if (resident * cols > 512) fail("tensor memory of the resident CTAs within 512 columns");
                if (b < (R == 16 ? psgd::TcSmem<16>::total : psgd::TcSmem<32>::total)) fail("tensor-core pass B buffers");
            }
        }
        if (sz.tiles != (int64_t)d.nrb * d.nchunk) fail("tile count");
    }
    // layer groups of the host-buffer steps (upload of later groups
    // overlapping the passes of earlier ones): 1..min(L, 8) groups, each a
    // non-empty contiguous layer range, every layer once, each group within
    // one layer of an equal share of the elements, and the groups' tile
    // ranges (the grids of their launches) following one another over the
    // whole grouped grid
    auto check_groups = [&](const char* name, const std::vector<std::pair<int64_t, int64_t>>& shapes, int r, int W) {
        psgd_ctx ctx;
        ctx.L = static_cast<int>(shapes.size());
        const int R = pad_rank(r);
        int64_t tiles = 0;
        double total = 0.0, biggest = 0.0;
        for (auto& sh : shapes) {
            LayerSizes sz{};
            LayerDesc d = layer_geometry(sh.first, sh.second, R, W, &sz);
            d.tile_begin = tiles;
            tiles += sz.tiles;
            ctx.desc.push_back(d);
            total += double(sh.first) * double(sh.second);
            biggest = std::max(biggest, double(sh.first) * double(sh.second));
        }
        const LayerGroups g = upload_groups(&ctx);
        ++n;
        auto gfail = [&](const char* what) {
            ++bad;
            std::printf("FAIL groups %s: %s (%zu groups)\n", name, what, g.size());
        };
        if (g.empty() || static_cast<int>(g.size()) > std::min(ctx.L, kUploadGroups)) gfail("1..min(L, 8) groups");
        int next = 0;
        int64_t tnext = 0;
        for (auto& lr : g) {
            const int l0 = lr.first, l1 = lr.second;
            if (l0 != next || l1 <= l0 || l1 > ctx.L) {
                gfail("contiguous, none empty");
                break;
            }
            double size = 0.0;
            for (int l = l0; l < l1; ++l) size += double(ctx.desc[l].m) * double(ctx.desc[l].n);
            if (size > total / double(g.size()) + biggest) gfail("within one layer of an equal share");
            const LayerDesc& last = ctx.desc[l1 - 1];
            const int64_t t0 = ctx.desc[l0].tile_begin, t1 = last.tile_begin + int64_t(last.nrb) * last.nchunk;
            if (t0 != tnext || t1 < t0) gfail("tile ranges follow one another");
            tnext = t1;
            next = l1;
        }
        if (next != ctx.L || tnext != tiles) gfail("every layer and tile once");
    };
    {
        std::vector<std::pair<int64_t, int64_t>> tf, rn, ls, mx, mx2;
        for (int b = 0; b < 24; ++b)
            for (auto& s2 : tf4) tf.push_back({s2[0], s2[1]});
        for (auto& s2 : resnet20) rn.push_back({s2[0], s2[1]});
        for (int k = 0; k < 6; ++k) ls.push_back({2600, 650});
        ls.push_back({33280, 650});
        ls.push_back({33280, 650});
        for (auto& s2 : mixed) mx.push_back({s2[0], s2[1]});
        mx2 = mx;
        mx2.insert(mx2.end(), mx.begin(), mx.end());
        check_groups("transformer set", tf, 4, 4);
        check_groups("ResNet-18 set", rn, 2, 16);
        check_groups("LSTM set", ls, 4, 16);
        check_groups("mixed shapes", mx, 4, 3);
        check_groups("mixed shapes twice", mx2, 4, 3);
        check_groups("one layer", {{300, 650}}, 4, 3);
        check_groups("small layers, one large last", {{8, 8}, {8, 8}, {8, 8}, {4096, 4096}}, 2, 2);
        check_groups("large first", {{4096, 4096}, {8, 8}, {8, 8}, {8, 8}, {8, 8}, {8, 8}, {8, 8}, {8, 8}, {8, 8}}, 2, 2);
    }
    std::printf("%d cases, %d failures\n", n, bad);
    return bad != 0;
}
