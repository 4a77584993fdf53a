// Three-axis position table (position_ids [3, B, L]) and rope deltas of a
// batch of mixed text / image / video sequences.
//
// "Interleaved Rotary Position Embedding" (taking-lying-flat.github.io),
// get_rope_index(): video grids are split into one (1, h, w) grid per temporal
// slice; one image and one video grid sequence serve the whole batch in order;
// per sample the padded slots are dropped, the kept slots are split into runs
// of equal type, and a running position walks the runs -- a text run takes
// consecutive positions on all three rows, a vision run lays its merged grid
// out width-fastest at (start + t, start + row, start + col) and moves the
// position on by its longer merged side.  The delta of a sample is its
// largest coordinate + 1 - its kept slot count.  Section "mm_tokens" gives the
// type codes (0 text, 1 image, 2 video, 3 audio); audio follows the text rule.
//
// The pages walk the runs one after another.  Here every coordinate follows
// from counts over the slots before it, which makes the table a scan:
//   * a kept text slot sits at (kept text slots before it in the sample)
//     + (advances of the sample's vision runs that start before it);
//   * a vision run starts at that same value and its k-th slot is the k-th
//     cell of its grid.
// Three launches, all on the caller's stream:
//   1. ri_tile_kernel   -- per tile of 1024 slots: kept / text counts, run
//      starts by kind, and where the last run start lies;
//   2. ri_carry_kernel  -- one block: the grid prefix sums, then per sample a
//      scan over its tiles giving the state before each tile (counts, the
//      summed advances, and the run still open at the tile's first slot);
//   3. ri_write_kernel  -- per tile: every slot's coordinates, the tile's
//      largest one, and in the last tile of a sample to finish, the delta.
// Slots of a kind the method does not define, grids that run out, and vision
// runs whose length differs from their grid's cell count are reported through
// the device status word (ipe_device_status); the table is still written.
#include <climits>

#include "ipe_internal.h"
#include "ipe_tma.cuh"

namespace ipe {

// Status codes of this kernel family (the word's first fault wins).
constexpr unsigned kRiNoGrid = 16;      // a vision run found no grid left
constexpr unsigned kRiRunLength = 17;   // a vision run's length differs from its grid's cell count
constexpr unsigned kRiBadType = 18;     // a kept slot of a type other than 0, 1, 2, 3
constexpr unsigned kRiBadGrid = 19;     // a grid with t, h or w outside 1 .. kRiMaxSide
constexpr unsigned kRiOverflow = 20;    // a coordinate beyond the int32 range
constexpr int kRiMaxSide = 1 << 15;

struct RiTileAgg {
    int kept, text;               // kept slots; kept text-like slots (type 0 or 3)
    int first_cls, last_cls;      // class of the first / last kept slot (-1: none)
    int img, vid;                 // image / video run starts, the first kept slot not counted
    int ls_off;                   // kept offset in the tile of the last such start (-1: none)
    int ls_text, ls_img, ls_vid;  // text slots and image / video starts of the tile before it
    int ls_cls, pad;
};

struct RiCarry {
    int k0, text0;                // kept and kept-text slots of the sample before the tile
    int img0, vid0;               // image / video runs of the batch before the tile
    long long vadv0;              // advances of the sample's vision runs started before the tile
    int prev_cls;                 // class of the last kept slot before the tile (-1: none)
    int open_k, open_grid;        // the run open at the tile's first slot: first kept index, grid
    int own_k, own_grid;          // the tile's own last run start (read by later tiles)
    int pad;
    long long open_start, own_start;
};

struct RiSample {
    int kept;                     // kept slots of the sample
    int img, vid;                 // image / video runs of the batch before the sample
    int max_pos;                  // largest coordinate written
    unsigned done;                // tiles finished
    int k_base, text_base;        // kept / kept-text slots of the batch before the sample
    int pad;
};

RopeIndexLayout rope_index_layout(long long B, long long L, int n_img, int n_vid)
{
    auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const long long tiles = B * ((L + kRiTile - 1) / kRiTile);
    RopeIndexLayout l;
    l.agg = up((size_t)tiles * sizeof(RiTileAgg));
    l.carry = up((size_t)tiles * sizeof(RiCarry));
    l.sample = up((size_t)B * sizeof(RiSample));
    l.img_adv = up((size_t)(n_img + 1) * sizeof(long long));
    l.vid_slices = up((size_t)(n_vid + 1) * sizeof(long long));
    l.vid_adv = up((size_t)(n_vid + 1) * sizeof(long long));
    l.total = l.agg + l.carry + l.sample + l.img_adv + l.vid_slices + l.vid_adv;
    return l;
}

// ------------------------------------------------------------------ access

__device__ __forceinline__ long long ld_int(const void *p, int bytes, long long i)
{
    return bytes == 8 ? static_cast<const long long *>(p)[i] : (long long)static_cast<const int *>(p)[i];
}

// Class of a slot: 0 text-like (types 0 and 3), 1 image, 2 video.  Types the
// method does not define are reported and laid out as text.
__device__ __forceinline__ void load_slots(const RopeIndexArgs &a, long long b, long long l0, int *cls, bool *kept,
                                           bool report)
{
#pragma unroll
    for (int i = 0; i < kRiPer; ++i) {
        const long long l = l0 + i;
        kept[i] = false;
        cls[i] = 0;
        if (l < a.L) {
            const long long at = b * a.L + l;
            kept[i] = a.mask == nullptr || ld_int(a.mask, a.id_bytes, at) != 0;
            const long long t = ld_int(a.types, a.id_bytes, at);
            if (t == 1 || t == 2) cls[i] = (int)t;
            else if (kept[i] && t != 0 && t != 3 && report) record_fault(a.status, kRiBadType);
        }
    }
}

struct RiGrid {
    int t, h, w;   // merged: t, h / merge, w / merge
    int adv;       // max(h, w) / merge
};

__device__ __forceinline__ bool side_ok(long long v) { return v >= 1 && v <= kRiMaxSide; }

// Grid row j of an image (t as given) or a video (t = 1 per slice).
__device__ __forceinline__ RiGrid grid_row(const RopeIndexArgs &a, const void *g, int j, bool video)
{
    const long long t = ld_int(g, a.grid_bytes, 3LL * j), h = ld_int(g, a.grid_bytes, 3LL * j + 1),
                    w = ld_int(g, a.grid_bytes, 3LL * j + 2);
    RiGrid r{0, 0, 0, 0};
    if (!side_ok(t) || !side_ok(h) || !side_ok(w)) return r;
    r.t = video ? 1 : (int)t;
    r.h = (int)h / a.merge;
    r.w = (int)w / a.merge;
    r.adv = (int)(h > w ? h : w) / a.merge;
    return r;
}

// Video grid row holding slice v (v below the slice total).
__device__ __forceinline__ int slice_row(const RopeIndexArgs &a, long long v)
{
    const long long *s = reinterpret_cast<const long long *>(a.vid_slices);
    int lo = 0, hi = a.n_vid - 1;   // the largest j with s[j] <= v
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Summed advances of the image grids [0, i) and of the video slices [0, v).
__device__ __forceinline__ long long img_adv_before(const RopeIndexArgs &a, long long i)
{
    return reinterpret_cast<const long long *>(a.img_adv)[i < a.n_img ? i : a.n_img];
}
__device__ __forceinline__ long long vid_adv_before(const RopeIndexArgs &a, long long v)
{
    const long long *s = reinterpret_cast<const long long *>(a.vid_slices);
    const long long *p = reinterpret_cast<const long long *>(a.vid_adv);
    if (a.n_vid == 0 || v >= s[a.n_vid]) return p[a.n_vid];
    const int j = slice_row(a, v);
    return p[j] + (v - s[j]) * (long long)grid_row(a, a.vid_grid, j, true).adv;
}

// Grid of vision run number g of class cls (false when the grids ran out).
__device__ __forceinline__ bool run_grid(const RopeIndexArgs &a, int cls, long long g, RiGrid &r)
{
    if (cls == 1) {
        if (g < 0 || g >= a.n_img) return false;
        r = grid_row(a, a.img_grid, (int)g, false);
        return true;
    }
    const long long *s = reinterpret_cast<const long long *>(a.vid_slices);
    if (g < 0 || a.n_vid == 0 || g >= s[a.n_vid]) return false;
    r = grid_row(a, a.vid_grid, slice_row(a, g), true);
    return true;
}

// ------------------------------------------------------------ block scans

// Four sums and a max (keys: 0 = none, larger = later).
struct RiSums {
    int kept, text, img, vid, last;
};

__device__ __forceinline__ RiSums ri_op(const RiSums &x, const RiSums &y)
{
    return {x.kept + y.kept, x.text + y.text, x.img + y.img, x.vid + y.vid, x.last > y.last ? x.last : y.last};
}

__device__ __forceinline__ RiSums ri_shfl_up(const RiSums &v, int d)
{
    return {__shfl_up_sync(0xffffffffu, v.kept, d), __shfl_up_sync(0xffffffffu, v.text, d),
            __shfl_up_sync(0xffffffffu, v.img, d), __shfl_up_sync(0xffffffffu, v.vid, d),
            __shfl_up_sync(0xffffffffu, v.last, d)};
}

// Exclusive scan over the block's threads in order; tot = the block total.
__device__ RiSums ri_block_exclusive(const RiSums &v, RiSums *warp_tot, RiSums &tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    RiSums inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const RiSums o = ri_shfl_up(inc, d);
        if (lane >= d) inc = ri_op(o, inc);
    }
    RiSums exc = ri_shfl_up(inc, 1);
    if (lane == 0) exc = RiSums{0, 0, 0, 0, 0};
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    RiSums pre{0, 0, 0, 0, 0};
    tot = pre;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        if (w < warp) pre = ri_op(pre, warp_tot[w]);
        tot = ri_op(tot, warp_tot[w]);
    }
    __syncthreads();
    return ri_op(pre, exc);
}

// ------------------------------------------------------- 1. tile aggregates

__global__ void __launch_bounds__(kRiThreads) ri_tile_kernel(const __grid_constant__ RopeIndexArgs a)
{
    __shared__ RiSums warp_tot[kRiThreads / 32];
    __shared__ RiTileAgg s;
    const long long tile = blockIdx.x;
    const long long b = tile / a.tiles_per_row;
    const int local0 = threadIdx.x * kRiPer;
    const long long l0 = (tile % a.tiles_per_row) * kRiTile + local0;
    int cls[kRiPer];
    bool kept[kRiPer];
    load_slots(a, b, l0, cls, kept, false);
    if (threadIdx.x == 0) s = RiTileAgg{0, 0, -1, -1, 0, 0, -1, 0, 0, 0, -1, 0};

    // class of the last kept slot before each thread's slots
    RiSums v{0, 0, 0, 0, 0}, tot1, tot2;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i)
        if (kept[i]) v.last = (local0 + i + 1) * 4 + cls[i];
    const RiSums ex1 = ri_block_exclusive(v, warp_tot, tot1);
    int prev = ex1.last ? (ex1.last & 3) : -1;

    // counts; run starts other than at the tile's first kept slot
    RiSums c{0, 0, 0, 0, 0};
    int ls_off = 0, ls_text = 0, ls_img = 0, ls_vid = 0, ls_cls = -1;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i) {
        if (!kept[i]) continue;
        if (prev < 0) {
            s.first_cls = cls[i];
        } else if (cls[i] != prev) {
            ls_off = c.kept;
            ls_text = c.text;
            ls_img = c.img;
            ls_vid = c.vid;
            ls_cls = cls[i];
            c.last = local0 + i + 1;
            c.img += cls[i] == 1;
            c.vid += cls[i] == 2;
        }
        c.kept += 1;
        c.text += cls[i] == 0;
        prev = cls[i];
    }
    const RiSums ex2 = ri_block_exclusive(c, warp_tot, tot2);
    if (c.last != 0 && c.last == tot2.last) {
        s.ls_off = ex2.kept + ls_off;
        s.ls_text = ex2.text + ls_text;
        s.ls_img = ex2.img + ls_img;
        s.ls_vid = ex2.vid + ls_vid;
        s.ls_cls = ls_cls;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        RiTileAgg o = s;
        o.kept = tot2.kept;
        o.text = tot2.text;
        o.img = tot2.img;
        o.vid = tot2.vid;
        o.last_cls = tot1.last ? (tot1.last & 3) : -1;
        static_cast<RiTileAgg *>(a.agg)[tile] = o;
    }
}

// --------------------------------------------------- 2. carries (one block)

constexpr int kRiCarryThreads = 1024;

// Exclusive block scan of long long pairs (1024 threads); tot = the total.
__device__ longlong2 scan_pair(longlong2 v, longlong2 *warp_tot, longlong2 &tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    longlong2 inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const long long x = __shfl_up_sync(0xffffffffu, inc.x, d), y = __shfl_up_sync(0xffffffffu, inc.y, d);
        if (lane >= d) {
            inc.x += x;
            inc.y += y;
        }
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    longlong2 pre{0, 0};
    tot = pre;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        if (w < warp) {
            pre.x += warp_tot[w].x;
            pre.y += warp_tot[w].y;
        }
        tot.x += warp_tot[w].x;
        tot.y += warp_tot[w].y;
    }
    __syncthreads();
    return make_longlong2(pre.x + inc.x - v.x, pre.y + inc.y - v.y);
}

// One thread per tile of the whole batch (in chunks of the block size), two
// block scans per chunk carried across chunks:
//   1. the latest tile with a kept slot (key (g + 1) * 4 + class, max):
//      the class before each tile, and whether its first kept slot starts a
//      run (the same sample only: the key's tile must not precede the
//      sample's first tile);
//   2. kept, text, image-run and video-run counts (sums over the batch) and
//      the latest tile with a run start (max).  Image / video runs of the
//      batch are plain prefix sums (the grid sequences serve the batch in
//      order); kept and text counts are taken relative to the sample's first
//      tile.
__global__ void __launch_bounds__(kRiCarryThreads) ri_carry_kernel(const __grid_constant__ RopeIndexArgs a)
{
    __shared__ longlong2 warp_tot2[kRiCarryThreads / 32];
    __shared__ RiSums warp_tot[kRiCarryThreads / 32];
    long long *img_adv = reinterpret_cast<long long *>(a.img_adv);
    long long *vid_slices = reinterpret_cast<long long *>(a.vid_slices);
    long long *vid_adv = reinterpret_cast<long long *>(a.vid_adv);
    RiSample *smp = static_cast<RiSample *>(a.sample);
    RiCarry *carry = static_cast<RiCarry *>(a.carry);
    const RiTileAgg *agg = static_cast<const RiTileAgg *>(a.agg);

    // grid prefix sums: image advances; video slices and slice advances
    longlong2 run{0, 0}, tot;
    for (int c0 = 0; c0 < a.n_img; c0 += blockDim.x) {
        const int j = c0 + threadIdx.x;
        long long adv = 0;
        if (j < a.n_img) {
            const long long t = ld_int(a.img_grid, a.grid_bytes, 3LL * j), h = ld_int(a.img_grid, a.grid_bytes, 3LL * j + 1),
                            w = ld_int(a.img_grid, a.grid_bytes, 3LL * j + 2);
            if (!side_ok(t) || !side_ok(h) || !side_ok(w)) record_fault(a.status, kRiBadGrid);
            adv = grid_row(a, a.img_grid, j, false).adv;
        }
        const longlong2 ex = scan_pair(make_longlong2(adv, 0), warp_tot2, tot);
        if (j < a.n_img) img_adv[j] = run.x + ex.x;
        run.x += tot.x;
    }
    if (threadIdx.x == 0) img_adv[a.n_img] = run.x;
    run = make_longlong2(0, 0);
    for (int c0 = 0; c0 < a.n_vid; c0 += blockDim.x) {
        const int j = c0 + threadIdx.x;
        longlong2 v{0, 0};
        if (j < a.n_vid) {
            const long long t = ld_int(a.vid_grid, a.grid_bytes, 3LL * j), h = ld_int(a.vid_grid, a.grid_bytes, 3LL * j + 1),
                            w = ld_int(a.vid_grid, a.grid_bytes, 3LL * j + 2);
            const bool good = side_ok(t) && side_ok(h) && side_ok(w);
            if (!good) record_fault(a.status, kRiBadGrid);
            v.x = good ? t : 0;
            v.y = v.x * grid_row(a, a.vid_grid, j, true).adv;
        }
        const longlong2 ex = scan_pair(v, warp_tot2, tot);
        if (j < a.n_vid) {
            vid_slices[j] = run.x + ex.x;
            vid_adv[j] = run.y + ex.y;
        }
        run.x += tot.x;
        run.y += tot.y;
    }
    if (threadIdx.x == 0) {
        vid_slices[a.n_vid] = run.x;
        vid_adv[a.n_vid] = run.y;
    }
    if (a.tiles_per_row == 0) {          // L = 0: no tiles, every delta is 0
        for (long long b = threadIdx.x; b < a.B; b += blockDim.x) a.deltas[b] = 0;
        return;
    }
    __syncthreads();

    const long long tiles = a.B * a.tiles_per_row;
    int run_last_kept = 0;
    RiSums run2{0, 0, 0, 0, 0};
    for (long long c0 = 0; c0 < tiles; c0 += blockDim.x) {
        const long long g = c0 + threadIdx.x;
        const bool valid = g < tiles;
        RiTileAgg r = RiTileAgg{0, 0, -1, -1, 0, 0, -1, 0, 0, 0, -1, 0};
        if (valid) r = agg[g];
        const long long b = valid ? g / a.tiles_per_row : 0;
        const long long g0 = b * a.tiles_per_row;
        const int t = (int)(g - g0);

        // 1. class of the last kept slot before the tile, within the sample
        RiSums v1{0, 0, 0, 0, r.kept > 0 ? (int)((g + 1) * 4 + r.last_cls) : 0}, tot1;
        RiSums ex1 = ri_block_exclusive(v1, warp_tot, tot1);
        const int key = max(ex1.last, run_last_kept);
        run_last_kept = max(run_last_kept, tot1.last);
        const int prev = (key > 0 && (key >> 2) - 1 >= g0) ? (key & 3) : -1;
        const bool fs = r.kept > 0 && r.first_cls != prev;
        const int img_t = r.img + (fs && r.first_cls == 1), vid_t = r.vid + (fs && r.first_cls == 2);
        const bool has = r.ls_off >= 0 || fs;

        // 2. counts over the batch and the latest tile with a run start
        RiSums v2{r.kept, r.text, img_t, vid_t, has ? (int)(g + 1) : 0}, tot2;
        const RiSums ex2 = ri_op(run2, ri_block_exclusive(v2, warp_tot, tot2));
        run2 = ri_op(run2, tot2);
        if (valid && t == 0) {
            smp[b].k_base = ex2.kept;
            smp[b].text_base = ex2.text;
            smp[b].img = ex2.img;
            smp[b].vid = ex2.vid;
        }
        __syncthreads();

        int k0 = 0, text0 = 0;
        long long base_adv = 0;
        if (valid) {
            const RiSample sm = smp[b];
            k0 = ex2.kept - sm.k_base;
            text0 = ex2.text - sm.text_base;
            base_adv = img_adv_before(a, sm.img) + vid_adv_before(a, sm.vid);
            // this tile's own last run start
            int own_k = 0, own_grid = -1;
            long long own_start = 0;
            if (has) {
                const bool fs_img = fs && r.first_cls == 1, fs_vid = fs && r.first_cls == 2;
                int off = 0, text_b = 0, ib = ex2.img, vb = ex2.vid, cls = r.first_cls;
                if (r.ls_off >= 0) {
                    off = r.ls_off;
                    text_b = r.ls_text;
                    ib = ex2.img + fs_img + r.ls_img;
                    vb = ex2.vid + fs_vid + r.ls_vid;
                    cls = r.ls_cls;
                }
                own_k = k0 + off;
                own_start = text0 + text_b + img_adv_before(a, ib) + vid_adv_before(a, vb) - base_adv;
                own_grid = cls == 1 ? ib : cls == 2 ? vb : -1;
            }
            carry[g].own_k = own_k;
            carry[g].own_grid = own_grid;
            carry[g].own_start = own_start;
        }
        __syncthreads();
        if (valid) {
            // the run open at the tile's first slot: the latest start before it, same sample
            const long long src = (long long)ex2.last - 1;
            const bool open = src >= g0;
            RiCarry &cr = carry[g];
            cr.k0 = k0;
            cr.text0 = text0;
            cr.img0 = ex2.img;
            cr.vid0 = ex2.vid;
            cr.vadv0 = img_adv_before(a, ex2.img) + vid_adv_before(a, ex2.vid) - base_adv;
            cr.prev_cls = prev;
            cr.open_k = open ? carry[src].own_k : 0;
            cr.open_grid = open ? carry[src].own_grid : -1;
            cr.open_start = open ? carry[src].own_start : 0;
            if (t == a.tiles_per_row - 1) {
                smp[b].kept = k0 + r.kept;
                smp[b].max_pos = -1;
                smp[b].done = 0u;
            }
        }
    }
}

// -------------------------------------------------------- 3. coordinates

__global__ void __launch_bounds__(kRiThreads) ri_write_kernel(const __grid_constant__ RopeIndexArgs a)
{
    __shared__ RiSums warp_tot[kRiThreads / 32];
    __shared__ int rec_k[kRiTile], rec_grid[kRiTile], rec_cls[kRiTile];
    __shared__ long long rec_start[kRiTile];
    __shared__ int warp_max[kRiThreads / 32];
    const long long tile = blockIdx.x;
    const long long b = tile / a.tiles_per_row;
    const int local0 = threadIdx.x * kRiPer;
    const long long l0 = (tile % a.tiles_per_row) * kRiTile + local0;
    const RiCarry C = static_cast<const RiCarry *>(a.carry)[tile];
    RiSample *smp = static_cast<RiSample *>(a.sample);
    const int sample_kept = smp[b].kept;
    const long long plane = a.B * a.L;
    int cls[kRiPer];
    bool kept[kRiPer];
    load_slots(a, b, l0, cls, kept, true);

    RiSums v{0, 0, 0, 0, 0}, tot;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i)
        if (kept[i]) v.last = (local0 + i + 1) * 4 + cls[i];
    const RiSums ex1 = ri_block_exclusive(v, warp_tot, tot);
    const int prev0 = ex1.last ? (ex1.last & 3) : C.prev_cls;

    // counts and run starts, the tile's first kept slot included
    RiSums c{0, 0, 0, 0, 0};
    int prev = prev0;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i) {
        if (!kept[i]) continue;
        if (cls[i] != prev) {
            c.last = local0 + i + 1;
            c.img += cls[i] == 1;
            c.vid += cls[i] == 2;
        }
        c.kept += 1;
        c.text += cls[i] == 0;
        prev = cls[i];
    }
    const RiSums ex = ri_block_exclusive(c, warp_tot, tot);

    // pass 1: records of the runs starting here; text slots
    long long vadv = C.vadv0 + img_adv_before(a, C.img0 + ex.img) - img_adv_before(a, C.img0) +
                     vid_adv_before(a, C.vid0 + ex.vid) - vid_adv_before(a, C.vid0);
    int kept_b = ex.kept, text_b = ex.text, img_b = ex.img, vid_b = ex.vid;
    long long mx = -1;
    prev = prev0;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i) {
        const long long l = l0 + i;
        if (l >= a.L) break;
        const long long at = b * a.L + l;
        if (!kept[i]) {
            a.pos[at] = 0;
            a.pos[plane + at] = 0;
            a.pos[2 * plane + at] = 0;
            continue;
        }
        const long long here = C.text0 + text_b + vadv;
        if (cls[i] != prev) {
            const int r = local0 + i;
            rec_k[r] = C.k0 + kept_b;
            rec_start[r] = here;
            rec_cls[r] = cls[i];
            rec_grid[r] = -1;
            if (cls[i] != 0) {
                const long long g = cls[i] == 1 ? (long long)C.img0 + img_b : (long long)C.vid0 + vid_b;
                RiGrid gr;
                rec_grid[r] = (int)g;
                if (run_grid(a, cls[i], g, gr)) vadv += gr.adv;
                img_b += cls[i] == 1;
                vid_b += cls[i] == 2;
            }
        }
        if (cls[i] == 0) {
            if (here > INT_MAX) record_fault(a.status, kRiOverflow);
            const int p = (int)min(here, (long long)INT_MAX);
            a.pos[at] = p;
            a.pos[plane + at] = p;
            a.pos[2 * plane + at] = p;
            mx = max(mx, (long long)p);
            ++text_b;
        }
        ++kept_b;
        prev = cls[i];
    }
    __syncthreads();

    // pass 2: vision slots from their run's record
    int rk = C.open_k, rgrid = C.open_grid, rcls = C.prev_cls > 0 ? C.prev_cls : 0;
    long long rstart = C.open_start;
    if (ex.last > 0) {
        const int r = ex.last - 1;
        rk = rec_k[r];
        rgrid = rec_grid[r];
        rcls = rec_cls[r];
        rstart = rec_start[r];
    }
    RiGrid gr{0, 0, 0, 0};
    bool have = rcls != 0 && run_grid(a, rcls, rgrid, gr);
    kept_b = ex.kept;
    prev = prev0;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i) {
        const long long l = l0 + i;
        if (l >= a.L) break;
        if (!kept[i]) continue;
        const int k = C.k0 + kept_b;
        if (cls[i] != prev) {
            // the run that ends here must have filled its grid
            if (rcls != 0 && (!have || (long long)(k - rk) != (long long)gr.t * gr.h * gr.w))
                record_fault(a.status, kRiRunLength);
            const int r = local0 + i;
            rk = rec_k[r];
            rgrid = rec_grid[r];
            rcls = rec_cls[r];
            rstart = rec_start[r];
            have = rcls != 0 && run_grid(a, rcls, rgrid, gr);
            if (rcls != 0 && !have) record_fault(a.status, kRiNoGrid);
        }
        if (cls[i] != 0) {
            const long long at = b * a.L + l;
            const long long off = k - rk;
            const long long cells = (long long)gr.t * gr.h * gr.w;
            long long tt = 0, row = 0, col = 0;
            if (have && off < cells) {
                const long long hw = (long long)gr.h * gr.w;
                tt = off / hw;
                const long long rem = off - tt * hw;
                row = rem / gr.w;
                col = rem - row * gr.w;
            } else if (have) {
                record_fault(a.status, kRiRunLength);
            }
            if (have && k == sample_kept - 1 && off + 1 != cells) record_fault(a.status, kRiRunLength);
            const long long pt = rstart + tt, ph = rstart + row, pw = rstart + col;
            const long long top = max(pt, max(ph, pw));
            if (top > INT_MAX) record_fault(a.status, kRiOverflow);
            a.pos[at] = (int)min(pt, (long long)INT_MAX);
            a.pos[plane + at] = (int)min(ph, (long long)INT_MAX);
            a.pos[2 * plane + at] = (int)min(pw, (long long)INT_MAX);
            mx = max(mx, min(top, (long long)INT_MAX));
        }
        ++kept_b;
        prev = cls[i];
    }

    // the tile's largest coordinate; the sample's last tile writes the delta
    int m = (int)mx;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kRiThreads / 32; ++w) m = max(m, warp_max[w]);
        if (m >= 0) atomicMax(&smp[b].max_pos, m);
        __threadfence();
        if (atomicAdd(&smp[b].done, 1u) == (unsigned)a.tiles_per_row - 1) {
            __threadfence();
            const int top = atomicAdd(&smp[b].max_pos, 0);
            a.deltas[b] = sample_kept > 0 ? top + 1 - sample_kept : 0;
        }
    }
}

cudaError_t launch_rope_index(const RopeIndexArgs &a, cudaStream_t s)
{
    const long long tiles = a.B * a.tiles_per_row;
    if (tiles > 0) ri_tile_kernel<<<(unsigned)tiles, kRiThreads, 0, s>>>(a);
    ri_carry_kernel<<<1, kRiCarryThreads, 0, s>>>(a);
    if (tiles > 0) ri_write_kernel<<<(unsigned)tiles, kRiThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ipe
