// Host-buffer entry points: the data moves host -> device, is processed and
// moves back in chunks, so that both copy directions and the kernels overlap.
//
// Per device the library keeps two copy streams (host-to-device and
// device-to-host, both non-blocking) and a ring of events.  A call splits its
// rows into chunks; for chunk c:
//   copies in   (h2d stream)  -> event in[c]
//   the kernel  (caller's stream, after in[c])  -> event done[c]
//   copies out  (d2h stream, after done[c])
// The copy streams are FIFO, so chunk c + 1 comes in while chunk c is
// processed and chunk c - 1 goes out.  Calls made one after another share
// the copy streams, so one call's copies overlap the next call's.
//
// Reuse of the caller's device buffers: the library remembers, per device
// buffer, the event after the last copy out of it; a later call waits on it
// before copying into that buffer again.  With join != 0 the caller's stream
// also waits for this call's copies out, so its completion means the
// results are in host memory; with join = 0 a later call with join != 0 (or
// ipe_host_join) gives that guarantee, for every earlier call on the device.
//
// Host buffers should be page-locked (cudaHostAlloc / pinned); pageable
// memory still works, but its copies do not overlap.
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "ipe.h"
#include "ipe_internal.h"

namespace ipe {
int set_error(int code, const char *msg);
}  // namespace ipe

namespace {

constexpr int kMaxDevices = 64;
constexpr int kRingEvents = 256;
constexpr int kBufferSlots = 64;

struct BufferSlot {
    const void *base;
    cudaEvent_t free_ev;     // recorded after the last copy out of the buffer
    unsigned long long age;
};

struct Pipe {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t ring[kRingEvents] = {};
    unsigned next = 0;
    BufferSlot slots[kBufferSlots] = {};
    unsigned long long clock = 0;
};

std::mutex g_pipe_mutex;
Pipe g_pipes[kMaxDevices];

int cuda_error(cudaError_t e, const char *what)
{
    char msg[256];
    snprintf(msg, sizeof msg, "%s: %s", what, cudaGetErrorString(e));
    cudaGetLastError();
    return ipe::set_error(IPE_ECUDA, msg);
}

#define IPE_TRY(call, what)                                  \
    do {                                                     \
        const cudaError_t e_ = (call);                       \
        if (e_ != cudaSuccess) return cuda_error(e_, what);  \
    } while (0)

// The pipe of the current device, created on first use (caller holds the lock).
int pipe_of_device(Pipe **out)
{
    int dev = -1;
    IPE_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return ipe::set_error(IPE_ELIMIT, "device index beyond 64");
    Pipe &p = g_pipes[dev];
    if (!p.ready) {
        IPE_TRY(cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking), "cudaStreamCreate (copies in)");
        IPE_TRY(cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking), "cudaStreamCreate (copies out)");
        for (int i = 0; i < kRingEvents; ++i)
            IPE_TRY(cudaEventCreateWithFlags(&p.ring[i], cudaEventDisableTiming), "cudaEventCreate");
        for (int i = 0; i < kBufferSlots; ++i)
            IPE_TRY(cudaEventCreateWithFlags(&p.slots[i].free_ev, cudaEventDisableTiming), "cudaEventCreate");
        p.ready = true;
    }
    *out = &p;
    return IPE_OK;
}

// A ring event: a wait enqueued on an event refers to the record made before
// it, so re-recording a ring entry later is safe.
cudaEvent_t ring_event(Pipe &p) { return p.ring[p.next++ % kRingEvents]; }

// Before copying into `base`: wait for the copies out of it of earlier calls.
int wait_buffer_free(Pipe &p, const void *base)
{
    for (BufferSlot &s : p.slots)
        if (s.base == base) {
            IPE_TRY(cudaStreamWaitEvent(p.h2d, s.free_ev, 0), "cudaStreamWaitEvent");
            break;
        }
    return IPE_OK;
}

// After the copies out of `base`: remember where they end.  When every slot
// is taken, the oldest is reused after the copies in wait for all copies out
// so far (nothing then depends on the forgotten entry).
int mark_buffer_used(Pipe &p, const void *base)
{
    BufferSlot *slot = nullptr, *oldest = &p.slots[0];
    for (BufferSlot &s : p.slots) {
        if (s.base == base) slot = &s;
        if (s.age < oldest->age) oldest = &s;
    }
    if (!slot) {
        for (BufferSlot &s : p.slots)
            if (s.base == nullptr) {
                slot = &s;
                break;
            }
    }
    if (!slot) {
        cudaEvent_t all = ring_event(p);
        IPE_TRY(cudaEventRecord(all, p.d2h), "cudaEventRecord");
        IPE_TRY(cudaStreamWaitEvent(p.h2d, all, 0), "cudaStreamWaitEvent");
        slot = oldest;
    }
    slot->base = base;
    slot->age = ++p.clock;
    IPE_TRY(cudaEventRecord(slot->free_ev, p.d2h), "cudaEventRecord");
    return IPE_OK;
}

// One chunk: copies in, the kernel on `s`, copies out.
struct Copy {
    void *dst;
    size_t dpitch;
    const void *src;
    size_t spitch, width, height;
};

// A copy as one linear transfer when its rows are contiguous on both sides.
cudaError_t copy_async(const Copy &c, cudaMemcpyKind kind, cudaStream_t s)
{
    if (c.dpitch == c.width && c.spitch == c.width) return cudaMemcpyAsync(c.dst, c.src, c.width * c.height, kind, s);
    return cudaMemcpy2DAsync(c.dst, c.dpitch, c.src, c.spitch, c.width, c.height, kind, s);
}

template <class Launch>
int run_chunk(Pipe &p, cudaStream_t s, const std::vector<Copy> &in, Launch launch, const std::vector<Copy> &out)
{
    for (const Copy &c : in)
        if (c.width && c.height) IPE_TRY(copy_async(c, cudaMemcpyHostToDevice, p.h2d), "copy in");
    cudaEvent_t ev_in = ring_event(p);
    IPE_TRY(cudaEventRecord(ev_in, p.h2d), "cudaEventRecord");
    IPE_TRY(cudaStreamWaitEvent(s, ev_in, 0), "cudaStreamWaitEvent");
    if (int rc = launch()) return rc;
    cudaEvent_t ev_done = ring_event(p);
    IPE_TRY(cudaEventRecord(ev_done, s), "cudaEventRecord");
    IPE_TRY(cudaStreamWaitEvent(p.d2h, ev_done, 0), "cudaStreamWaitEvent");
    for (const Copy &c : out)
        if (c.width && c.height) IPE_TRY(copy_async(c, cudaMemcpyDeviceToHost, p.d2h), "copy out");
    return IPE_OK;
}

// The caller's stream waits for every copy out enqueued so far.
int join_stream(Pipe &p, cudaStream_t s)
{
    cudaEvent_t ev = ring_event(p);
    IPE_TRY(cudaEventRecord(ev, p.d2h), "cudaEventRecord");
    IPE_TRY(cudaStreamWaitEvent(s, ev, 0), "cudaStreamWaitEvent");
    return IPE_OK;
}

// Work of one call, with the buffer bookkeeping around it.
template <class Body>
int pipelined(const std::vector<const void *> &buffers, int join, cudaStream_t s, Body body)
{
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    Pipe *p = nullptr;
    if (int rc = pipe_of_device(&p)) return rc;
    // the caller's earlier work on `s` comes before this call's copies in
    cudaEvent_t start = ring_event(*p);
    IPE_TRY(cudaEventRecord(start, s), "cudaEventRecord");
    IPE_TRY(cudaStreamWaitEvent(p->h2d, start, 0), "cudaStreamWaitEvent");
    for (const void *b : buffers)
        if (b)
            if (int rc = wait_buffer_free(*p, b)) return rc;
    if (int rc = body(*p)) return rc;
    for (const void *b : buffers)
        if (b)
            if (int rc = mark_buffer_used(*p, b)) return rc;
    return join ? join_stream(*p, s) : IPE_OK;
}

size_t elem_size(ipe_dtype dt) { return dt == IPE_BF16 ? 2 : 4; }

// Vision chunks: whole images grouped up to chunk_rows patches; an image
// above that is split into frame ranges (its frames share one layout).
struct VisChunk {
    std::vector<int32_t> grid;    // sub-grid rows (t, h, w)
    long long row0, rows;         // patch rows of the whole call
};

std::vector<VisChunk> vis_chunks(const int32_t *grid, int n_images, long long chunk_rows)
{
    std::vector<VisChunk> out;
    VisChunk cur{{}, 0, 0};
    long long row = 0;
    for (int i = 0; i < n_images; ++i) {
        const long long t = grid[3 * i], h = grid[3 * i + 1], w = grid[3 * i + 2], hw = h * w;
        if (t * hw <= chunk_rows) {
            if (cur.rows + t * hw > chunk_rows && cur.rows > 0) {
                out.push_back(cur);
                cur = VisChunk{{}, row, 0};
            }
            if (cur.rows == 0) cur.row0 = row;
            cur.grid.insert(cur.grid.end(), {(int32_t)t, (int32_t)h, (int32_t)w});
            cur.rows += t * hw;
        } else {
            if (cur.rows > 0) {
                out.push_back(cur);
                cur = VisChunk{{}, 0, 0};
            }
            const long long fpc = hw > 0 ? (chunk_rows / hw > 0 ? chunk_rows / hw : 1) : 1;
            for (long long f = 0; f < t; f += fpc) {
                const long long k = t - f < fpc ? t - f : fpc;
                out.push_back(VisChunk{{(int32_t)k, (int32_t)h, (int32_t)w}, row + f * hw, k * hw});
            }
        }
        row += t * hw;
    }
    if (cur.rows > 0) out.push_back(cur);
    return out;
}

}  // namespace

extern "C" {

int ipe_host_join(void *stream)
{
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    Pipe *p = nullptr;
    if (int rc = pipe_of_device(&p)) return rc;
    return join_stream(*p, (cudaStream_t)stream);
}

int ipe_mrope_apply_host(const void *q_host, const void *k_host, void *q_out_host, void *k_out_host, ipe_dtype dtype,
                         int64_t T, int hq, int hk, int head_dim, const int32_t *positions_host,
                         const float *inv_freq_host, int rot_dim, const int32_t *section, int interleaved,
                         void *q_dev, void *k_dev, int32_t *positions_dev, int64_t chunk_tokens, int join,
                         void *stream)
{
    if (chunk_tokens < 1) return ipe::set_error(IPE_EINVAL, "chunk_tokens must be >= 1");
    if (T < 0 || hq < 0 || hk < 0 || head_dim < 1) return ipe::set_error(IPE_EINVAL, "bad sizes");
    if (T > 0 && (!positions_host || !positions_dev || (hq && (!q_host || !q_out_host || !q_dev)) ||
                  (hk && (!k_host || !k_out_host || !k_dev))))
        return ipe::set_error(IPE_EINVAL, "a buffer is NULL");
    const size_t eb = elem_size(dtype);
    const size_t qrow = (size_t)hq * head_dim * eb, krow = (size_t)hk * head_dim * eb;
    // In place (out == in), channels past rot_dim never change: only the
    // rotary slice of each head row crosses the link, as a strided copy
    // (rows of rot_dim elements, pitch head_dim), into the same place of the
    // staging buffer.  Otherwise whole token rows move.
    const bool slices = q_out_host == q_host && k_out_host == k_host && rot_dim > 0 && rot_dim < head_dim;
    const size_t hrow = (size_t)head_dim * eb, srow = slices ? (size_t)rot_dim * eb : hrow;
    cudaStream_t s = (cudaStream_t)stream;
    return pipelined({q_dev, k_dev, positions_dev}, join, s, [&](Pipe &p) -> int {
        for (long long t0 = 0; t0 < T; t0 += chunk_tokens) {
            const long long n = T - t0 < chunk_tokens ? T - t0 : chunk_tokens;
            char *dq = static_cast<char *>(q_dev) + t0 * qrow, *dk = static_cast<char *>(k_dev) + t0 * krow;
            int32_t *dpos = positions_dev + 3 * t0;   // this chunk's positions, [3, n]
            const size_t nq = hq ? (size_t)n * hq : 0, nk = hk ? (size_t)n * hk : 0;   // head rows
            std::vector<Copy> in = {
                {dq, hrow, static_cast<const char *>(q_host) + t0 * qrow, hrow, srow, nq},
                {dk, hrow, static_cast<const char *>(k_host) + t0 * krow, hrow, srow, nk},
                {dpos, (size_t)n * 4, positions_host + t0, (size_t)T * 4, (size_t)n * 4, 3},
            };
            std::vector<Copy> out = {
                {static_cast<char *>(q_out_host) + t0 * qrow, hrow, dq, hrow, srow, nq},
                {static_cast<char *>(k_out_host) + t0 * krow, hrow, dk, hrow, srow, nk},
            };
            int rc = run_chunk(p, s, in, [&]() {
                return ipe_mrope_apply(hq ? dq : nullptr, hk ? dk : nullptr, dtype, n, hq, hk, head_dim,
                                       (int64_t)hq * head_dim, (int64_t)hk * head_dim, dpos, inv_freq_host, rot_dim,
                                       section, interleaved, stream);
            }, out);
            if (rc) return rc;
        }
        return IPE_OK;
    });
}

int ipe_vis_rope2d_host(const void *q_host, const void *k_host, void *q_out_host, void *k_out_host, ipe_dtype dtype,
                        int heads, int head_dim, const int32_t *grid_thw_host, int n_images, int merge, double theta,
                        void *q_dev, void *k_dev, int64_t chunk_rows, int join, void *stream)
{
    if (chunk_rows < 1) return ipe::set_error(IPE_EINVAL, "chunk_rows must be >= 1");
    if (heads < 1 || head_dim < 1 || n_images < 0 || (n_images > 0 && !grid_thw_host))
        return ipe::set_error(IPE_EINVAL, "bad sizes");
    for (int i = 0; i < 3 * n_images; ++i)
        if (grid_thw_host[i] < 1) return ipe::set_error(IPE_EINVAL, "grid_thw has a non-positive size");
    if (!q_host || !q_out_host || !q_dev || (k_dev && (!k_host || !k_out_host)))
        return ipe::set_error(IPE_EINVAL, "a buffer is NULL");
    const size_t row = (size_t)heads * head_dim * elem_size(dtype);
    const std::vector<VisChunk> chunks = vis_chunks(grid_thw_host, n_images, chunk_rows);
    cudaStream_t s = (cudaStream_t)stream;
    return pipelined({q_dev, k_dev}, join, s, [&](Pipe &p) -> int {
        for (const VisChunk &c : chunks) {
            char *dq = static_cast<char *>(q_dev) + c.row0 * row;
            char *dk = k_dev ? static_cast<char *>(k_dev) + c.row0 * row : nullptr;
            std::vector<Copy> in = {{dq, row, static_cast<const char *>(q_host) + c.row0 * row, row, row, (size_t)c.rows}};
            std::vector<Copy> out = {{static_cast<char *>(q_out_host) + c.row0 * row, row, dq, row, row, (size_t)c.rows}};
            if (dk) {
                in.push_back({dk, row, static_cast<const char *>(k_host) + c.row0 * row, row, row, (size_t)c.rows});
                out.push_back({static_cast<char *>(k_out_host) + c.row0 * row, row, dk, row, row, (size_t)c.rows});
            }
            int rc = run_chunk(p, s, in, [&]() {
                return ipe_vis_rope2d(dq, dk, dtype, c.rows, heads, head_dim, (int64_t)heads * head_dim,
                                      (int64_t)heads * head_dim, c.grid.data(), (int)(c.grid.size() / 3), merge, theta,
                                      stream);
            }, out);
            if (rc) return rc;
        }
        return IPE_OK;
    });
}

int ipe_vis_pos_interp_host(const void *table_host, ipe_dtype dtype, int grid_side, int hidden,
                            const int32_t *grid_thw_host, int n_images, int merge, void *out_host, void *table_dev,
                            void *out_dev, int64_t chunk_rows, int join, void *stream)
{
    if (chunk_rows < 1) return ipe::set_error(IPE_EINVAL, "chunk_rows must be >= 1");
    if (grid_side < 1 || hidden < 1 || n_images < 0 || (n_images > 0 && !grid_thw_host))
        return ipe::set_error(IPE_EINVAL, "bad sizes");
    for (int i = 0; i < 3 * n_images; ++i)
        if (grid_thw_host[i] < 1) return ipe::set_error(IPE_EINVAL, "grid_thw has a non-positive size");
    if (!table_host || !table_dev || !out_host || !out_dev) return ipe::set_error(IPE_EINVAL, "a buffer is NULL");
    const size_t row = (size_t)hidden * elem_size(dtype);
    const size_t table_bytes = (size_t)grid_side * grid_side * row;
    const std::vector<VisChunk> chunks = vis_chunks(grid_thw_host, n_images, chunk_rows);
    cudaStream_t s = (cudaStream_t)stream;
    return pipelined({table_dev, out_dev}, join, s, [&](Pipe &p) -> int {
        bool first = true;
        for (const VisChunk &c : chunks) {
            char *dout = static_cast<char *>(out_dev) + c.row0 * row;
            std::vector<Copy> in;
            if (first) in.push_back({table_dev, table_bytes, table_host, table_bytes, table_bytes, 1});
            first = false;
            std::vector<Copy> out = {{static_cast<char *>(out_host) + c.row0 * row, row, dout, row, row, (size_t)c.rows}};
            int rc = run_chunk(p, s, in, [&]() {
                return ipe_vis_pos_interp(table_dev, dtype, grid_side, hidden, c.grid.data(), (int)(c.grid.size() / 3),
                                          merge, dout, stream);
            }, out);
            if (rc) return rc;
        }
        return IPE_OK;
    });
}

}  // extern "C"
