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
// One kernel on the caller's stream, after a memset of the tile flags, the
// per-sample records and the tile ticket:
//   ri_scan_kernel -- one block per tile of 1024 slots, in the order the
//   blocks start (a ticket), as a single-pass scan with decoupled
//   look-back: the block publishes its tile's own counts, looks back to the
//   nearest earlier tile that has published its inclusive state, folds the
//   counts of the tiles in between onto it (32 tiles per warp step),
//   publishes its own inclusive state, then writes every slot's
//   coordinates; the last tile of a sample to finish writes the delta.  The
//   block with the first ticket also writes the grid prefix sums (image
//   advances, video slices and slice advances) and flags them ready; the
//   others wait for that flag before their write pass.
// Every wait is bounded: a tile that gives up records code 23 in the device
// status word and marks itself failed, so that the tiles waiting on it give
// up at once instead of waiting out their own limit.
// Slots of a kind the method does not define, grids that run out, and vision
// runs whose length differs from their grid's cell count are reported through
// the device status word (ipe_device_status); the table is still written.
#include <climits>

#include "ipe_internal.h"
#include "ipe_rotary.cuh"
#include "ipe_tma.cuh"

namespace ipe {

// Status codes of this kernel family (the word's first fault wins).
constexpr unsigned kRiNoGrid = 16;      // a vision run found no grid left
constexpr unsigned kRiRunLength = 17;   // a vision run's length differs from its grid's cell count
constexpr unsigned kRiBadType = 18;     // a kept slot of a type other than 0, 1, 2, 3
constexpr unsigned kRiBadGrid = 19;     // a grid with t, h or w outside 1 .. kRiMaxSide
constexpr unsigned kRiOverflow = 20;    // a coordinate beyond the int32 range
constexpr unsigned kRiLookback = 23;    // a tile gave up waiting for an earlier tile's counts
constexpr int kRiMaxSide = 1 << 15;

// Publication flag of a tile (cleared by ri_init_kernel); it only grows.
constexpr unsigned kRiNone = 0;         // nothing yet
constexpr unsigned kRiAgg = 1;          // the tile's own counts (RiTileAgg)
constexpr unsigned kRiPrefix = 2;       // ... and the inclusive state after it (RiState)
constexpr unsigned kRiFailed = 3;       // the tile gave up: nothing will follow

struct RiTileAgg {
    int kept, text;               // kept slots; kept text-like slots (type 0 or 3)
    int first_cls, last_cls;      // class of the first / last kept slot (-1: none)
    int img, vid;                 // image / video run starts, the first kept slot not counted
    int ls_off;                   // kept offset in the tile of the last such start (-1: none)
    int ls_text, ls_img, ls_vid;  // text slots and image / video starts of the tile before it
    int ls_cls, pad;
};

// What the tiles of the batch up to and including one tile leave for the
// next tile.  The latest run start keeps its grid indices, not its first
// position, so that folding tiles needs no grid look-ups.
struct RiState {
    int K, TX;                     // kept / kept text-like slots of the current sample
    int IMG, VID;                  // image / video runs of the batch
    int IMGB, VIDB;                // image / video runs of the batch before the current sample
    int PC;                        // class of the sample's last kept slot (-1: none)
    int open_cls;                  // class of the sample's latest run (-1: none)
    int open_k, open_tx;           // its first kept index; the text slots of the sample before it
    int open_ib, open_vb;          // image / video runs of the batch before it
};

struct RiSample {
    int kept;                      // kept slots of the sample (written by its last tile)
    int max_pos1;                  // largest coordinate written + 1 (0: none)
    unsigned done;                 // tiles finished
    int tail_bad1;                 // kept index + 1 of a tile-final vision slot whose run is incomplete (0: none)
};

RopeIndexLayout rope_index_layout(long long B, long long L, int n_img, int n_vid)
{
    auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const long long tiles = B * ((L + kRiTile - 1) / kRiTile);
    RopeIndexLayout l;
    l.agg = up((size_t)tiles * sizeof(RiTileAgg));
    l.state = up((size_t)tiles * sizeof(RiState));
    l.flags = up((size_t)tiles * sizeof(unsigned));
    l.sample = up((size_t)B * sizeof(RiSample));
    l.ticket = 256;
    l.img_adv = up((size_t)(n_img + 1) * sizeof(long long));
    l.vid_slices = up((size_t)(n_vid + 1) * sizeof(long long));
    l.vid_adv = up((size_t)(n_vid + 1) * sizeof(long long));
    l.total = l.agg + l.state + l.flags + l.sample + l.ticket + l.img_adv + l.vid_slices + l.vid_adv;
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

// ------------------------------------------------- grid prefix sums (init)


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

// The grid prefix sums (image advances, video slices and slice advances),
// written by the block that takes the first ticket; the others wait for
// `ready` before their write pass.
__device__ void ri_grid_prefix(const RopeIndexArgs &a, longlong2 *warp_tot2)
{
    long long *img_adv = a.img_adv, *vid_slices = a.vid_slices, *vid_adv = a.vid_adv;
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
}

// ------------------------------------------------------------ look-back

__device__ __forceinline__ unsigned ld_flag(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_flag(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ RiState ri_start_state()
{
    return RiState{0, 0, 0, 0, 0, 0, -1, -1, 0, 0, 0, 0};
}

// A sample begins: its counts, class and latest run start the empty ones.
__device__ __forceinline__ void ri_begin_sample(RiState &x)
{
    x.K = 0;
    x.TX = 0;
    x.PC = -1;
    x.IMGB = x.IMG;
    x.VIDB = x.VID;
    x.open_cls = -1;
    x.open_k = x.open_tx = x.open_ib = x.open_vb = 0;
}

// The state after a tile from the state before it (a sample's first tile
// already begun) and the tile's own counts.  The tile's first kept slot
// starts a run when its class differs from the sample's last kept class.
__device__ __forceinline__ void ri_fold(RiState &x, const RiTileAgg &r)
{
    const bool fs = r.kept > 0 && r.first_cls != x.PC;
    const int fs_img = fs && r.first_cls == 1, fs_vid = fs && r.first_cls == 2;
    if (r.ls_off >= 0) {               // the tile's latest run start lies past its first kept slot
        x.open_k = x.K + r.ls_off;
        x.open_tx = x.TX + r.ls_text;
        x.open_ib = x.IMG + fs_img + r.ls_img;
        x.open_vb = x.VID + fs_vid + r.ls_vid;
        x.open_cls = r.ls_cls;
    } else if (fs) {                   // ... or is its first kept slot
        x.open_k = x.K;
        x.open_tx = x.TX;
        x.open_ib = x.IMG;
        x.open_vb = x.VID;
        x.open_cls = r.first_cls;
    }
    x.K += r.kept;
    x.TX += r.text;
    x.IMG += r.img + fs_img;
    x.VID += r.vid + fs_vid;
    if (r.kept > 0) x.PC = r.last_cls;
}

__device__ __forceinline__ RiTileAgg ld_agg(const RiTileAgg *p)
{
    const int4 *q = reinterpret_cast<const int4 *>(p);
    const int4 u = __ldcg(q), v = __ldcg(q + 1), w = __ldcg(q + 2);
    return RiTileAgg{u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w, w.x, w.y, w.z, w.w};
}

__device__ __forceinline__ RiState ld_state(const RiState *p)
{
    const int4 *q = reinterpret_cast<const int4 *>(p);
    const int4 u = __ldcg(q), v = __ldcg(q + 1), w = __ldcg(q + 2);
    return RiState{u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w, w.x, w.y, w.z, w.w};
}

__device__ __forceinline__ int warp_incl_sum(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += t;
    }
    return v;
}

__device__ __forceinline__ int warp_incl_max(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v = max(v, t);
    }
    return v;
}

// Warp: fold the counts of tiles c .. c + n - 1 (1 <= n <= 32, lane i holds
// tile c + i) onto x, the state after tile c - 1 (the same in every lane).
// The folds of ri_fold, done for the window at once:
//   * the class before each tile: the latest earlier tile of the window with
//     a kept slot in the same sample (a max-scan of keys), else x's class,
//     else none when the tile's sample starts inside the window;
//   * whether each tile's first kept slot starts a run, hence its image /
//     video run starts;
//   * kept and text counts, reset at sample starts, and the batch's image
//     and video run counts (sum-scans);
//   * the latest run start of the last tile's sample (a max-scan).
__device__ void ri_fold_window(const RopeIndexArgs &a, RiState &x, long long c, int n)
{
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const bool valid = lane < n;
    const RiTileAgg r = valid ? ld_agg(static_cast<const RiTileAgg *>(a.agg) + c + lane)
                              : RiTileAgg{0, 0, -1, -1, 0, 0, -1, 0, 0, 0, -1, 0};
    const bool start = valid && (c + lane) % a.tiles_per_row == 0;
    const int ss = warp_incl_max(start ? lane : -1);           // this tile's sample start in the window (-1: before it)
    const int kinc = warp_incl_max(valid && r.kept > 0 ? (lane + 1) * 4 + r.last_cls : 0);
    int kex = __shfl_up_sync(full, kinc, 1);
    if (lane == 0) kex = 0;
    const int prev = (kex > 0 && (kex >> 2) - 1 >= ss) ? (kex & 3) : (ss < 0 ? x.PC : -1);
    const bool fs = valid && r.kept > 0 && r.first_cls != prev;
    const int fi = fs && r.first_cls == 1, fv = fs && r.first_cls == 2;
    const int img_t = r.img + fi, vid_t = r.vid + fv;
    const int pk = warp_incl_sum(r.kept) - r.kept, ptx = warp_incl_sum(r.text) - r.text;
    const int pimg = warp_incl_sum(img_t) - img_t, pvid = warp_incl_sum(vid_t) - vid_t;
    const int src = ss < 0 ? 0 : ss;
    const int pk_s = __shfl_sync(full, pk, src), ptx_s = __shfl_sync(full, ptx, src);
    const int pimg_s = __shfl_sync(full, pimg, src), pvid_s = __shfl_sync(full, pvid, src);
    // values before this lane's tile
    const int K0 = ss < 0 ? x.K + pk : pk - pk_s;
    const int TX0 = ss < 0 ? x.TX + ptx : ptx - ptx_s;
    const int IMG0 = x.IMG + pimg, VID0 = x.VID + pvid;
    const int IMGB = ss < 0 ? x.IMGB : x.IMG + pimg_s, VIDB = ss < 0 ? x.VIDB : x.VID + pvid_s;
    // this tile's latest run start
    int ok = 0, otx = 0, oib = 0, ovb = 0, ocls = -1;
    if (valid && r.ls_off >= 0) {
        ok = K0 + r.ls_off;
        otx = TX0 + r.ls_text;
        oib = IMG0 + fi + r.ls_img;
        ovb = VID0 + fv + r.ls_vid;
        ocls = r.ls_cls;
    } else if (fs) {
        ok = K0;
        otx = TX0;
        oib = IMG0;
        ovb = VID0;
        ocls = r.first_cls;
    }
    const int hj = warp_incl_max(ocls >= 0 ? lane : -1);
    // the state after the window's last tile
    const int L = n - 1;
    RiState y;
    y.K = __shfl_sync(full, K0 + r.kept, L);
    y.TX = __shfl_sync(full, TX0 + r.text, L);
    y.IMG = __shfl_sync(full, IMG0 + img_t, L);
    y.VID = __shfl_sync(full, VID0 + vid_t, L);
    y.IMGB = __shfl_sync(full, IMGB, L);
    y.VIDB = __shfl_sync(full, VIDB, L);
    y.PC = __shfl_sync(full, r.kept > 0 ? r.last_cls : prev, L);
    const int ssL = __shfl_sync(full, ss, L), hL = __shfl_sync(full, hj, L);
    const int hs = hL < 0 ? 0 : hL;
    const int ok_h = __shfl_sync(full, ok, hs), otx_h = __shfl_sync(full, otx, hs);
    const int oib_h = __shfl_sync(full, oib, hs), ovb_h = __shfl_sync(full, ovb, hs);
    const int ocls_h = __shfl_sync(full, ocls, hs);
    if (hL >= 0 && hL >= ssL) {                    // a run starts in the last tile's sample, in the window
        y.open_k = ok_h;
        y.open_tx = otx_h;
        y.open_ib = oib_h;
        y.open_vb = ovb_h;
        y.open_cls = ocls_h;
    } else if (ssL < 0) {                          // the sample continues from x with no new run
        y.open_k = x.open_k;
        y.open_tx = x.open_tx;
        y.open_ib = x.open_ib;
        y.open_vb = x.open_vb;
        y.open_cls = x.open_cls;
    } else {                                       // the sample started in the window with no run yet
        y.open_k = y.open_tx = y.open_ib = y.open_vb = 0;
        y.open_cls = -1;
    }
    x = y;
}

// Warp 0: the state before tile `tile` (of the whole batch so far; the
// caller begins the sample when the tile is a sample's first).  Looks back
// 32 tiles at a time for the nearest tile with its inclusive state
// published, every tile in between having published its counts, then folds
// those counts onto it, 32 tiles per step.  False when a wait ran out or an
// earlier tile failed.
__device__ bool ri_look_back(const RopeIndexArgs &a, long long tile, RiState &out)
{
    const int lane = threadIdx.x & 31;
    const RiState *st = static_cast<const RiState *>(a.state);
    const long long t0 = clock64();
    long long hi = tile - 1, p = -1;   // p: the tile whose state starts the fold (-1: the batch start)
    while (hi >= 0) {
        const long long j = hi - lane;
        unsigned f = kRiPrefix;        // before the batch start: the empty state
        if (j >= 0) {
            f = ld_flag(a.flags + j);
            while (f == kRiNone && clock64() - t0 <= a.wait_limit) f = ld_flag(a.flags + j);
        }
        // lane l reads tile hi - l: lanes below the nearest prefix are the
        // tiles after it, whose counts the fold needs
        const unsigned bad = __ballot_sync(0xffffffffu, f == kRiNone || f == kRiFailed);
        const unsigned pre = __ballot_sync(0xffffffffu, f == kRiPrefix);
        if (pre) {
            const int l = __ffs(pre) - 1;
            if (bad & ((1u << l) - 1u)) return false;
            p = hi - l;
            break;
        }
        if (bad) return false;
        hi -= 32;
    }
    // every lane reads data that other lanes saw published
    __syncwarp();
    __threadfence();
    RiState x = p >= 0 ? ld_state(st + p) : ri_start_state();
    for (long long c = p + 1; c < tile; c += 32) ri_fold_window(a, x, c, (int)min(32LL, tile - c));
    out = x;
    return true;
}

// ------------------------------------------------------------- the scan

__global__ void __launch_bounds__(kRiThreads) ri_scan_kernel(const __grid_constant__ RopeIndexArgs a)
{
    __shared__ RiSums warp_tot[kRiThreads / 32];
    __shared__ RiTileAgg s;
    __shared__ RiState before;
    __shared__ long long tile_sh;
    __shared__ int ok_sh;
    __shared__ int rec_k[kRiTile], rec_grid[kRiTile], rec_cls[kRiTile];
    __shared__ long long rec_start[kRiTile];
    __shared__ int warp_max[kRiThreads / 32];

    // tiles in the order the blocks start, so every tile waited on is running
    __shared__ longlong2 warp_tot2[kRiThreads / 32];
    if (threadIdx.x == 0) tile_sh = (long long)atomicAdd(a.ticket, 1u);
    __syncthreads();
    const long long tile = tile_sh;
    if (tile == 0) {
        ri_grid_prefix(a, warp_tot2);
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            st_flag(a.ticket + 1, 1u);
        }
    }
    if (tile == a.skip_tile) return;   // test hook: this tile never publishes anything
    const long long b = tile / a.tiles_per_row;
    const int t_in_row = (int)(tile % a.tiles_per_row);
    const int local0 = threadIdx.x * kRiPer;
    const long long l0 = (long long)t_in_row * kRiTile + local0;
    int cls[kRiPer];
    bool kept[kRiPer];
    load_slots(a, b, l0, cls, kept, true);

    // ---- the tile's own counts, nothing before it known
    if (threadIdx.x == 0) s = RiTileAgg{0, 0, -1, -1, 0, 0, -1, 0, 0, 0, -1, 0};
    RiSums v{0, 0, 0, 0, 0}, tot1, tot2;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i)
        if (kept[i]) v.last = (local0 + i + 1) * 4 + cls[i];
    const RiSums ex1 = ri_block_exclusive(v, warp_tot, tot1);
    const int prev_in_tile = ex1.last ? (ex1.last & 3) : -1;   // last kept class before this thread's slots
    {
        RiSums c{0, 0, 0, 0, 0};
        int prev = prev_in_tile;
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
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s.kept = tot2.kept;
        s.text = tot2.text;
        s.img = tot2.img;
        s.vid = tot2.vid;
        s.last_cls = tot1.last ? (tot1.last & 3) : -1;
        static_cast<RiTileAgg *>(a.agg)[tile] = s;
        st_flag(a.flags + tile, kRiAgg);
    }

    // ---- the state before the tile, then the state after it
    if (threadIdx.x < 32) {
        RiState x;
        const bool ok = ri_look_back(a, tile, x);
        if (threadIdx.x == 0) {
            ok_sh = ok;
            if (ok) {
                if (t_in_row == 0) ri_begin_sample(x);
                before = x;
                ri_fold(x, s);
                static_cast<RiState *>(a.state)[tile] = x;
                st_flag(a.flags + tile, kRiPrefix);
                if (t_in_row == a.tiles_per_row - 1) static_cast<RiSample *>(a.sample)[b].kept = x.K;
            } else {
                record_fault(a.status, kRiLookback);
                st_flag(a.flags + tile, kRiFailed);
            }
        }
    }
    if (threadIdx.x == 0 && ok_sh) {
        // the grid prefix sums of the first tile's block
        const long long t0 = clock64();
        unsigned r = ld_flag(a.ticket + 1);
        while (r == 0u && clock64() - t0 <= a.wait_limit) r = ld_flag(a.ticket + 1);
        if (r == 0u) {
            record_fault(a.status, kRiLookback);
            ok_sh = 0;
        }
    }
    __syncthreads();
    if (!ok_sh) return;
    const RiState X = before;
    RiSample *smp = static_cast<RiSample *>(a.sample);
    const long long plane = a.B * a.L;
    const long long base_adv = img_adv_before(a, X.IMGB) + vid_adv_before(a, X.VIDB);
    const long long vadv0 = img_adv_before(a, X.IMG) + vid_adv_before(a, X.VID) - base_adv;

    // ---- counts and run starts with the class before the tile known
    const int prev0 = ex1.last ? (ex1.last & 3) : X.PC;
    RiSums c{0, 0, 0, 0, 0}, tot;
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
    long long vadv = vadv0 + img_adv_before(a, X.IMG + ex.img) - img_adv_before(a, X.IMG) +
                     vid_adv_before(a, X.VID + ex.vid) - vid_adv_before(a, X.VID);
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
        const long long here = X.TX + text_b + vadv;
        if (cls[i] != prev) {
            const int r = local0 + i;
            rec_k[r] = X.K + kept_b;
            rec_start[r] = here;
            rec_cls[r] = cls[i];
            rec_grid[r] = -1;
            if (cls[i] != 0) {
                const long long g = cls[i] == 1 ? (long long)X.IMG + img_b : (long long)X.VID + vid_b;
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

    // pass 2: vision slots from their run's record (or the run open at the
    // tile's first slot)
    int rk = X.open_cls >= 0 ? X.open_k : 0;
    int rgrid = X.open_cls == 1 ? X.open_ib : X.open_cls == 2 ? X.open_vb : -1;
    int rcls = X.PC > 0 ? X.PC : 0;
    long long rstart = X.open_cls >= 0 ? X.open_tx + img_adv_before(a, X.open_ib) + vid_adv_before(a, X.open_vb) - base_adv
                                       : 0;
    if (ex.last > 0) {
        const int r = ex.last - 1;
        rk = rec_k[r];
        rgrid = rec_grid[r];
        rcls = rec_cls[r];
        rstart = rec_start[r];
    }
    RiGrid gr{0, 0, 0, 0};
    bool have = rcls != 0 && run_grid(a, rcls, rgrid, gr);
    const int tile_last = tot1.last ? (tot1.last >> 2) - 1 : -1;   // local index of the tile's last kept slot
    kept_b = ex.kept;
    prev = prev0;
#pragma unroll
    for (int i = 0; i < kRiPer; ++i) {
        const long long l = l0 + i;
        if (l >= a.L) break;
        if (!kept[i]) continue;
        const int k = X.K + kept_b;
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
            // a run still short of its grid at the tile's last kept slot: a
            // fault if that slot turns out to be the sample's last
            if (have && local0 + i == tile_last && off + 1 != cells) atomicMax(&smp[b].tail_bad1, k + 1);
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

    // the tile's largest coordinate; the sample's last tile to finish writes the delta
    int m = (int)mx;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kRiThreads / 32; ++w) m = max(m, warp_max[w]);
        if (m >= 0) atomicMax(&smp[b].max_pos1, m + 1);
        __threadfence();
        if (atomicAdd(&smp[b].done, 1u) == (unsigned)a.tiles_per_row - 1) {
            __threadfence();
            const int kept_n = __ldcg(&smp[b].kept);
            const int top = atomicAdd(&smp[b].max_pos1, 0) - 1;
            const int bad = atomicAdd(&smp[b].tail_bad1, 0) - 1;
            if (kept_n > 0 && bad == kept_n - 1) record_fault(a.status, kRiRunLength);
            a.deltas[b] = kept_n > 0 ? top + 1 - kept_n : 0;
        }
    }
}

cudaError_t launch_rope_index(const RopeIndexArgs &a, cudaStream_t s)
{
    const long long tiles = a.B * a.tiles_per_row;
    if (tiles == 0) return cudaMemsetAsync(a.deltas, 0, (size_t)a.B * sizeof(int32_t), s);   // L = 0
    // flags, sample records and ticket are one contiguous run of the workspace
    const size_t zero = (size_t)(reinterpret_cast<char *>(a.ticket) - reinterpret_cast<char *>(a.flags)) + 256;
    cudaError_t e = cudaMemsetAsync(a.flags, 0, zero, s);
    if (e != cudaSuccess) return e;
    ri_scan_kernel<<<(unsigned)tiles, kRiThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ipe
