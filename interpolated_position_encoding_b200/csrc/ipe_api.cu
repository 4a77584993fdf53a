// C ABI of libipe.so: argument validation, descriptor packing and launches on
// the caller's stream.  See include/ipe.h for the contract of every entry
// point.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <cuda.h>   // CUresult / CUdeviceptr types only; the driver call is resolved at run time

#include "ipe.h"
#include "ipe_internal.h"
#include "ipe_rotary_tma.cuh"

using namespace ipe;

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok()
{
    g_err.clear();
    return IPE_OK;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(IPE_ECUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

// cuMemGetAddressRange through the runtime's driver entry point (no link
// dependency on libcuda, so the library loads on machines without a GPU).
typedef CUresult (*AddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);

AddressRangeFn address_range_fn()
{
    // resolved once (thread-safe static initialisation)
    static const AddressRangeFn fn = []() -> AddressRangeFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<AddressRangeFn>(p);
        cudaGetLastError();
        return nullptr;
    }();
    return fn;
}

// `p` must be device (or managed) memory of the current device whose
// allocation covers [p, p + bytes).
int check_dev(const void *p, size_t bytes, const char *name)
{
    if (bytes == 0) return IPE_OK;
    if (p == nullptr) return fail(IPE_EINVAL, "%s is NULL", name);
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, name);
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return fail(IPE_EINVAL, "%s is not device memory", name);
    int dev = -1;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (at.type == cudaMemoryTypeDevice && at.device != dev)
        return fail(IPE_EINVAL, "%s lives on device %d, current device is %d", name, at.device, dev);
    if (AddressRangeFn fn = address_range_fn()) {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (fn(&base, &size, (CUdeviceptr)(uintptr_t)p) == CUDA_SUCCESS) {
            const uintptr_t end = (uintptr_t)base + size;
            if ((uintptr_t)p + bytes > end || (uintptr_t)p + bytes < (uintptr_t)p)
                return fail(IPE_EINVAL, "%s: %zu bytes from the pointer run past its allocation (%zu bytes left)",
                            name, bytes, (size_t)(end - (uintptr_t)p));
        }
    }
    return IPE_OK;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// ------------------------------------------------- status word, test hooks
__device__ unsigned g_ipe_status;     // first fault code of any kernel since the last read

long long g_skip_tile = -1;
long long g_wait_limit = 0;           // 0: default
constexpr long long kDefaultWaitCycles = 1LL << 31;   // about 1.1 s at 1.9 GHz

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn()
{
    // resolved once (thread-safe static initialisation)
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
        return nullptr;
    }();
    return fn;
}

int elem_bytes(ipe_dtype dt) { return dt == IPE_BF16 ? 2 : 4; }

int check_dtype(int dt)
{
    if (dt != IPE_F32 && dt != IPE_BF16) return fail(IPE_EINVAL, "dtype %d is neither IPE_F32 nor IPE_BF16", dt);
    return IPE_OK;
}

int check_section(int half, const int32_t *section)
{
    if (section == nullptr) return fail(IPE_EINVAL, "section is NULL");
    if (section[0] < 0 || section[1] < 0 || section[2] < 0)
        return fail(IPE_EINVAL, "mrope_section (%d, %d, %d) has a negative count", section[0], section[1], section[2]);
    if ((long long)section[0] + section[1] + section[2] != half)
        return fail(IPE_EINVAL, "mrope_section (%d, %d, %d) sums to %lld, not rot_dim/2 = %d", section[0],
                    section[1], section[2], (long long)section[0] + section[1] + section[2], half);
    return IPE_OK;
}

int check_half(int half)
{
    if (half < 1) return fail(IPE_EINVAL, "rot_dim/2 = %d must be >= 1", half);
    if (half > IPE_MAX_HALF) return fail(IPE_ELIMIT, "rot_dim/2 = %d is above IPE_MAX_HALF = %d", half, IPE_MAX_HALF);
    return IPE_OK;
}

// Bytes spanned by `rows` rows of `heads` heads of `head_dim` elements.
size_t span_bytes(long long rows, long long stride, int heads, int head_dim, int eb)
{
    if (rows <= 0 || heads <= 0) return 0;
    return (size_t)(((rows - 1) * stride + (long long)heads * head_dim) * eb);
}

// Head-row tensors of a rotation call.
int check_qk(void *q, void *k, ipe_dtype dt, long long rows, int hq, int hk, int head_dim, long long qs,
             long long ks, const char *qn, const char *kn)
{
    if (rows < 0) return fail(IPE_EINVAL, "row count %lld is negative", rows);
    if (hq < 0 || hk < 0) return fail(IPE_EINVAL, "head counts (%d, %d) must be >= 0", hq, hk);
    if (head_dim <= 0) return fail(IPE_EINVAL, "head_dim %d must be > 0", head_dim);
    if (hq > 0 && qs < (long long)hq * head_dim)
        return fail(IPE_EINVAL, "%s row stride %lld < heads * head_dim = %lld", qn, qs, (long long)hq * head_dim);
    if (hk > 0 && ks < (long long)hk * head_dim)
        return fail(IPE_EINVAL, "%s row stride %lld < heads * head_dim = %lld", kn, ks, (long long)hk * head_dim);
    if (rows > 0 && hq > 0 && q == nullptr) return fail(IPE_EINVAL, "%s is NULL but has %d heads", qn, hq);
    if (rows > 0 && hk > 0 && k == nullptr) return fail(IPE_EINVAL, "%s is NULL but has %d heads", kn, hk);
    const int eb = elem_bytes(dt);
    if (!aligned(q, eb) || !aligned(k, eb)) return fail(IPE_EALIGN, "%s / %s not aligned to the element size", qn, kn);
    if (hq > 0) {
        if (int rc = check_dev(q, span_bytes(rows, qs, hq, head_dim, eb), qn)) return rc;
    }
    if (hk > 0) {
        if (int rc = check_dev(k, span_bytes(rows, ks, hk, head_dim, eb), kn)) return rc;
    }
    if (rows > 0 && (long long)(hq + hk) * head_dim > (1LL << 30))
        return fail(IPE_ELIMIT, "heads * head_dim too large");
    return IPE_OK;
}

// Vision descriptor from host grid_thw.
int build_vis_desc(const int32_t *grid, int n_images, int merge, int grid_side, VisDesc<1024> &d)
{
    if (grid == nullptr && n_images > 0) return fail(IPE_EINVAL, "grid_thw is NULL");
    if (n_images < 0) return fail(IPE_EINVAL, "n_images %d is negative", n_images);
    if (n_images > IPE_MAX_IMAGES)
        return fail(IPE_ELIMIT, "n_images %d is above IPE_MAX_IMAGES = %d", n_images, IPE_MAX_IMAGES);
    if (merge < 1 || merge > 8) return fail(IPE_EINVAL, "merge %d must be in 1 .. 8", merge);
    if (grid_side < 1 || grid_side > 256) return fail(IPE_EINVAL, "grid_side %d must be in 1 .. 256", grid_side);
    d.n_images = n_images;
    d.merge = merge;
    d.grid_side = grid_side;
    long long row = 0;
    long long strips = 0;
    for (int i = 0; i < n_images; ++i) {
        const int t = grid[3 * i], h = grid[3 * i + 1], w = grid[3 * i + 2];
        if (t < 1 || h < 1 || w < 1)
            return fail(IPE_EINVAL, "grid_thw[%d] = (%d, %d, %d) has a non-positive size", i, t, h, w);
        if (h % merge || w % merge)
            return fail(IPE_EINVAL, "grid_thw[%d] = (%d, %d, %d): h and w must be multiples of merge %d", i, t, h,
                        w, merge);
        if (h > 65536 || w > 65536 || t > 65536)
            return fail(IPE_ELIMIT, "grid_thw[%d] = (%d, %d, %d): sides above 65536", i, t, h, w);
        d.img[i].t = t;
        d.img[i].h = h;
        d.img[i].w = w;
        d.img[i].strip0 = (int)strips;
        d.img[i].row0 = row;
        row += (long long)t * h * w;
        strips += h / merge;
    }
    if (row > (1LL << 31) - 1) return fail(IPE_ELIMIT, "more than 2^31 - 1 patches");
    if (strips > (1LL << 24)) return fail(IPE_ELIMIT, "too many merge-row strips");
    d.n_patch = row;
    d.n_strips = (int)strips;
    return IPE_OK;
}

int vis_freqs(int head_dim, double theta, VisAngleFreqs &f)
{
    if (head_dim <= 0 || head_dim % 4) return fail(IPE_EINVAL, "vision head_dim %d must be a positive multiple of 4", head_dim);
    if (head_dim / 4 > kMaxVisFreq) return fail(IPE_ELIMIT, "vision head_dim %d above %d", head_dim, 4 * kMaxVisFreq);
    if (!(theta > 0.0) || !std::isfinite(theta)) return fail(IPE_EINVAL, "theta must be finite and > 0");
    const int dim = head_dim / 2;
    f.nf = head_dim / 4;
    for (int i = 0; i < f.nf; ++i) f.inv[i] = (float)(1.0 / std::pow(theta, (double)(2 * i) / (double)dim));
    return IPE_OK;
}

// Per-thread host buffer of the vision descriptor (about 25 KB).
VisDesc<1024> *desc_buffer()
{
    thread_local VisDesc<1024> *dp = nullptr;
    if (!dp) dp = new VisDesc<1024>();
    return dp;
}

}  // namespace

namespace ipe {

unsigned *device_status_word()
{
    static unsigned *addr[64] = {};
    static std::mutex lock_addr;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> guard(lock_addr);   // callers on several host threads
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ipe_status) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = static_cast<unsigned *>(p);
    }
    return addr[dev];
}

long long debug_skip_tile() { return g_skip_tile; }
long long debug_wait_limit() { return g_wait_limit > 0 ? g_wait_limit : kDefaultWaitCycles; }

bool encode_tmap(CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                 const uint64_t *strides, const uint32_t *box)
{
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn || rank < 1 || rank > 3 || !aligned(base, 16)) return false;
    cuuint64_t gdim[3], gstr[2];
    cuuint32_t bdim[3], estr[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        if (dims[i] == 0 || dims[i] > (1ULL << 32) || box[i] == 0 || box[i] > 256) return false;
        gdim[i] = dims[i];
        bdim[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) {
        if (strides[i] % 16 || strides[i] >= (1ULL << 40)) return false;
        gstr[i] = strides[i];
    }
    return fn(map, dt, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstr, bdim, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tma_rot_args(const RotArgs &r, int eb, TmaRotArgs &t)
{
    const int rot = 2 * r.half;
    if ((rot * eb) % 16 || rot > 256 || (r.head_dim * eb) % 16) return false;
    if (r.hq > 256 || r.hk > 256 || r.rows <= 0 || r.rows > 0x7fffffffLL) return false;
    // one stage (P rows of q and k) must stay far below the shared memory and
    // the 2^20-byte transaction count of a barrier phase
    if ((size_t)kTmaRows * (r.hq + r.hk) * rot * eb > 96 * 1024) return false;
    const CUtensorMapDataType dt = eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    t = TmaRotArgs{};
    t.P = kTmaRows;
    struct Side {
        CUtensorMap *tile, *one;
        void *ptr;
        int heads;
        long long stride;
    } sides[2] = {{&t.tq, &t.tq1, r.q, r.hq, r.q_stride}, {&t.tk, &t.tk1, r.k, r.hk, r.k_stride}};
    for (const Side &sd : sides) {
        if (!sd.heads) continue;
        const uint64_t dims[3] = {(uint64_t)r.head_dim, (uint64_t)sd.heads, (uint64_t)r.rows};
        const uint64_t str[2] = {(uint64_t)r.head_dim * eb, (uint64_t)sd.stride * eb};
        const uint32_t box_tile[3] = {(uint32_t)rot, (uint32_t)sd.heads, (uint32_t)t.P};
        const uint32_t box_one[3] = {(uint32_t)rot, (uint32_t)sd.heads, 1};
        if (!encode_tmap(sd.tile, dt, 3, sd.ptr, dims, str, box_tile)) return false;
        if (!encode_tmap(sd.one, dt, 3, sd.ptr, dims, str, box_one)) return false;
    }
    t.rows = r.rows;
    t.hq = r.hq;
    t.hk = r.hk;
    t.half = r.half;
    t.wait_limit = debug_wait_limit();
    t.skip_tile = debug_skip_tile();
    t.status = device_status_word();
    return t.status != nullptr;
}

// Status and message for ipe_last_error, for entry points in other files.
int set_error(int code, const char *msg) { return fail(code, "%s", msg); }

}  // namespace ipe

extern "C" {

const char *ipe_last_error(void) { return g_err.c_str(); }

int ipe_version(void) { return 100; }

int ipe_kernel_arch(int *binary_version, int *ptx_version)
{
    if (binary_version == nullptr || ptx_version == nullptr) return fail(IPE_EINVAL, "output pointer is NULL");
    cudaFuncAttributes attr{};
    cudaError_t e = mrope_axis_map_attributes(&attr);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
    *binary_version = attr.binaryVersion;
    *ptx_version = attr.ptxVersion;
    return ok();
}

int ipe_device_status(void *stream)
{
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_ipe_status, sizeof v)) != cudaSuccess) return cuda_fail(e, "status read");
    if (v == 0) return ok();
    const unsigned zero = 0;
    if ((e = cudaMemcpyToSymbol(g_ipe_status, &zero, sizeof zero)) != cudaSuccess) return cuda_fail(e, "status clear");
    const char *what = v == 1 ? "a consumer warp gave up waiting for a stage's data"
                     : v == 2 ? "the producer gave up waiting for a free stage"
                     : v == 3 ? "loads in flight did not land while a block shut down"
                     : v == 16 ? "position table: a vision run found no grid left"
                     : v == 17 ? "position table: a vision run's length differs from its grid's cell count"
                     : v == 18 ? "position table: a kept slot has a type other than 0, 1, 2, 3"
                     : v == 19 ? "position table: a grid has t, h or w outside 1 .. 32768"
                     : v == 20 ? "position table: a coordinate beyond the int32 range"
                     : v == 21 ? "decode: seq_pos + rope delta outside [0, 2^24)"
                     : v == 22 ? "decode: a cache slot at or beyond num_slots (that write was skipped)"
                     : v == 23 ? "position table: a tile gave up waiting for an earlier tile's counts"
                              : "unknown";
    return fail(IPE_EDEVICE, "device fault %u: %s", v, what);
}

int ipe_debug_inject(int64_t skip_tile, int64_t wait_cycles)
{
    if (wait_cycles < 0) return fail(IPE_EINVAL, "wait_cycles %lld is negative", (long long)wait_cycles);
    g_skip_tile = skip_tile < 0 ? -1 : skip_tile;
    g_wait_limit = wait_cycles;
    return ok();
}

int ipe_rope_inv_freq(int rot_dim, double theta, float *inv_freq_host)
{
    if (rot_dim < 2 || rot_dim % 2) return fail(IPE_EINVAL, "rot_dim %d must be even and >= 2", rot_dim);
    if (rot_dim / 2 > IPE_MAX_HALF) return fail(IPE_ELIMIT, "rot_dim %d above 2*IPE_MAX_HALF", rot_dim);
    if (!(theta > 0.0) || !std::isfinite(theta)) return fail(IPE_EINVAL, "theta must be finite and > 0");
    if (inv_freq_host == nullptr) return fail(IPE_EINVAL, "inv_freq_host is NULL");
    for (int j = 0; j < rot_dim / 2; ++j)
        inv_freq_host[j] = (float)(1.0 / std::pow(theta, (double)(2 * j) / (double)rot_dim));
    return ok();
}

int ipe_mrope_axis_map(int half, const int32_t *section, int interleaved, int8_t *axis_dev, void *stream)
{
    if (int rc = check_half(half)) return rc;
    if (int rc = check_section(half, section)) return rc;
    if (int rc = check_dev(axis_dev, (size_t)half, "axis_dev")) return rc;
    cudaError_t e = launch_mrope_axis_map(half, section, interleaved ? 1 : 0, axis_dev, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "mrope_axis_map launch");
}

static int fill_mrope(MropeAngles &a, const int32_t *positions, int64_t T, const float *inv, int half,
                      const int32_t *section, int interleaved)
{
    if (T < 0) return fail(IPE_EINVAL, "T = %lld is negative", (long long)T);
    if (T > (1LL << 40)) return fail(IPE_ELIMIT, "T = %lld too large", (long long)T);
    if (int rc = check_half(half)) return rc;
    if (int rc = check_section(half, section)) return rc;
    if (inv == nullptr) return fail(IPE_EINVAL, "inv_freq_host is NULL");
    for (int j = 0; j < half; ++j)
        if (!std::isfinite(inv[j])) return fail(IPE_EINVAL, "inv_freq[%d] is not finite", j);
    if (T > 0 && !aligned(positions, 4)) return fail(IPE_EALIGN, "positions not 4-byte aligned");
    a.positions = positions;
    a.T = T;
    a.section[0] = section[0];
    a.section[1] = section[1];
    a.section[2] = section[2];
    a.interleaved = interleaved ? 1 : 0;
    for (int j = 0; j < half; ++j) a.inv[j] = inv[j];
    for (int j = half; j < kMaxHalf; ++j) a.inv[j] = 0.f;
    return IPE_OK;
}

int ipe_mrope_cos_sin(const int32_t *positions, int64_t T, const float *inv_freq_host, int half,
                      const int32_t *section, int interleaved, float *cos_out, float *sin_out, void *stream)
{
    MropeAngles a;
    if (int rc = fill_mrope(a, positions, T, inv_freq_host, half, section, interleaved)) return rc;
    if (T == 0) return ok();
    if (!aligned(cos_out, 4) || !aligned(sin_out, 4)) return fail(IPE_EALIGN, "cos_out / sin_out not 4-byte aligned");
    if (int rc = check_dev(positions, (size_t)(3 * T) * 4, "positions")) return rc;
    if (int rc = check_dev(cos_out, (size_t)T * 2 * half * 4, "cos_out")) return rc;
    if (int rc = check_dev(sin_out, (size_t)T * 2 * half * 4, "sin_out")) return rc;
    cudaError_t e = launch_mrope_cos_sin(a, half, cos_out, sin_out, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "mrope_cos_sin launch");
}

static int apply_rotary_partial_impl(bool hf, void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk,
                                     int head_dim, int64_t q_tok_stride, int64_t k_tok_stride, const float *cos,
                                     const float *sin, int rot_dim, void *stream)
{
    if (int rc = check_dtype(dtype)) return rc;
    if (rot_dim < 2 || rot_dim % 2) return fail(IPE_EINVAL, "rot_dim %d must be even and >= 2", rot_dim);
    if (int rc = check_half(rot_dim / 2)) return rc;
    if (rot_dim > head_dim) return fail(IPE_EINVAL, "rot_dim %d > head_dim %d", rot_dim, head_dim);
    if (int rc = check_qk(q, k, dtype, T, hq, hk, head_dim, q_tok_stride, k_tok_stride, "q", "k")) return rc;
    if (T == 0 || hq + hk == 0) return ok();
    if (!aligned(cos, 4) || !aligned(sin, 4)) return fail(IPE_EALIGN, "cos / sin not 4-byte aligned");
    if (int rc = check_dev(cos, (size_t)T * rot_dim * 4, "cos")) return rc;
    if (int rc = check_dev(sin, (size_t)T * rot_dim * 4, "sin")) return rc;
    RotArgs r{};
    r.q = hq ? q : nullptr;
    r.k = hk ? k : nullptr;
    r.rows = T;
    r.q_stride = q_tok_stride;
    r.k_stride = k_tok_stride;
    r.hq = hq;
    r.hk = hk;
    r.head_dim = head_dim;
    r.half = rot_dim / 2;
    TableAngles a{cos, sin};
    cudaError_t e = launch_rotary_table(dtype == IPE_BF16, r, a, (cudaStream_t)stream, hf);
    return e == cudaSuccess ? ok() : cuda_fail(e, "apply_rotary_partial launch");
}

int ipe_apply_rotary_partial(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                             int64_t q_tok_stride, int64_t k_tok_stride, const float *cos, const float *sin,
                             int rot_dim, void *stream)
{
    return apply_rotary_partial_impl(false, q, k, dtype, T, hq, hk, head_dim, q_tok_stride, k_tok_stride, cos, sin,
                                     rot_dim, stream);
}

int ipe_apply_rotary_partial_hf(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                                int64_t q_tok_stride, int64_t k_tok_stride, const float *cos, const float *sin,
                                int rot_dim, void *stream)
{
    return apply_rotary_partial_impl(true, q, k, dtype, T, hq, hk, head_dim, q_tok_stride, k_tok_stride, cos, sin,
                                     rot_dim, stream);
}

static int mrope_apply_impl(bool hf, void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                            int64_t q_tok_stride, int64_t k_tok_stride, const int32_t *positions,
                            const float *inv_freq_host, int rot_dim, const int32_t *section, int interleaved,
                            void *stream)
{
    if (int rc = check_dtype(dtype)) return rc;
    if (rot_dim < 2 || rot_dim % 2) return fail(IPE_EINVAL, "rot_dim %d must be even and >= 2", rot_dim);
    if (rot_dim > head_dim) return fail(IPE_EINVAL, "rot_dim %d > head_dim %d", rot_dim, head_dim);
    MropeAngles a;
    if (int rc = fill_mrope(a, positions, T, inv_freq_host, rot_dim / 2, section, interleaved)) return rc;
    if (int rc = check_qk(q, k, dtype, T, hq, hk, head_dim, q_tok_stride, k_tok_stride, "q", "k")) return rc;
    if (T == 0 || hq + hk == 0) return ok();
    if (int rc = check_dev(positions, (size_t)(3 * T) * 4, "positions")) return rc;
    RotArgs r{};
    r.q = hq ? q : nullptr;
    r.k = hk ? k : nullptr;
    r.rows = T;
    r.q_stride = q_tok_stride;
    r.k_stride = k_tok_stride;
    r.hq = hq;
    r.hk = hk;
    r.head_dim = head_dim;
    r.half = rot_dim / 2;
    cudaError_t e = launch_rotary_mrope(dtype == IPE_BF16, r, a, (cudaStream_t)stream, hf);
    return e == cudaSuccess ? ok() : cuda_fail(e, "mrope_apply launch");
}

int ipe_mrope_apply(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                    int64_t q_tok_stride, int64_t k_tok_stride, const int32_t *positions, const float *inv_freq_host,
                    int rot_dim, const int32_t *section, int interleaved, void *stream)
{
    return mrope_apply_impl(false, q, k, dtype, T, hq, hk, head_dim, q_tok_stride, k_tok_stride, positions,
                            inv_freq_host, rot_dim, section, interleaved, stream);
}

int ipe_mrope_apply_hf(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim,
                       int64_t q_tok_stride, int64_t k_tok_stride, const int32_t *positions,
                       const float *inv_freq_host, int rot_dim, const int32_t *section, int interleaved, void *stream)
{
    return mrope_apply_impl(true, q, k, dtype, T, hq, hk, head_dim, q_tok_stride, k_tok_stride, positions,
                            inv_freq_host, rot_dim, section, interleaved, stream);
}

int ipe_qk_norm_mrope(void *q, void *k, ipe_dtype dtype, int64_t T, int hq, int hk, int head_dim, int64_t q_tok_stride,
                      int64_t k_tok_stride, const void *q_weight, const void *k_weight, float eps,
                      const int32_t *positions, const float *inv_freq_host, int rot_dim, const int32_t *section,
                      int interleaved, void *stream)
{
    if (int rc = check_dtype(dtype)) return rc;
    const int eb = elem_bytes(dtype), ec = 16 / eb;
    if (head_dim <= 0 || head_dim % ec) return fail(IPE_EINVAL, "head_dim %d must be a multiple of %d", head_dim, ec);
    const int lpr = head_dim / ec;
    if (lpr < 2 || lpr > 32 || (lpr & (lpr - 1)))
        return fail(IPE_ELIMIT, "head_dim %d: %d-element chunks per row must be a power of two in 2 .. 32", head_dim, ec);
    if (rot_dim < 2 || rot_dim % 2 || rot_dim > head_dim)
        return fail(IPE_EINVAL, "rot_dim %d must be even and in 2 .. head_dim", rot_dim);
    if ((rot_dim / 2) % ec) return fail(IPE_EINVAL, "rot_dim / 2 = %d must be a multiple of %d", rot_dim / 2, ec);
    if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(IPE_EINVAL, "eps must be finite and >= 0");
    MropeAngles a;
    if (int rc = fill_mrope(a, positions, T, inv_freq_host, rot_dim / 2, section, interleaved)) return rc;
    if (int rc = check_qk(q, k, dtype, T, hq, hk, head_dim, q_tok_stride, k_tok_stride, "q", "k")) return rc;
    if ((hq && (q_tok_stride % ec || !aligned(q, 16))) || (hk && (k_tok_stride % ec || !aligned(k, 16))))
        return fail(IPE_EALIGN, "q / k and their token strides must be 16-byte aligned");
    if (!aligned(q_weight, 16) || !aligned(k_weight, 16)) return fail(IPE_EALIGN, "norm weights must be 16-byte aligned");
    if (T == 0 || hq + hk == 0) return ok();
    if (int rc = check_dev(q_weight, (size_t)head_dim * eb, "q_weight")) return rc;
    if (int rc = check_dev(k_weight, (size_t)head_dim * eb, "k_weight")) return rc;
    if (int rc = check_dev(positions, (size_t)(3 * T) * 4, "positions")) return rc;
    QkNormArgs n{};
    n.q = hq ? q : nullptr;
    n.k = hk ? k : nullptr;
    n.q_weight = q_weight;
    n.k_weight = k_weight;
    n.T = T;
    n.q_stride = q_tok_stride;
    n.k_stride = k_tok_stride;
    n.hq = hq;
    n.hk = hk;
    n.head_dim = head_dim;
    n.half = rot_dim / 2;
    n.half_pad = (n.half + 3) & ~3;
    n.eps = eps;
    cudaError_t e = launch_qk_norm_mrope(dtype == IPE_BF16, n, a, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "qk_norm_mrope launch");
}

int ipe_mrope_decode(void *q, void *k, const void *v, ipe_dtype dtype, int64_t B, int hq, int hk, int head_dim,
                     int64_t q_tok_stride, int64_t k_tok_stride, int64_t v_tok_stride, const int32_t *seq_pos,
                     const int32_t *rope_deltas, const void *q_weight, const void *k_weight, float eps,
                     const float *inv_freq_host, int rot_dim, void *k_cache, void *v_cache, int64_t cache_slot_stride,
                     int64_t num_slots, const int64_t *slot_mapping, void *stream)
{
    if (int rc = check_dtype(dtype)) return rc;
    const int eb = elem_bytes(dtype), ec = 16 / eb;
    if (head_dim <= 0 || head_dim % ec) return fail(IPE_EINVAL, "head_dim %d must be a multiple of %d", head_dim, ec);
    const int lpr = head_dim / ec;
    if (lpr < 2 || lpr > 32 || (lpr & (lpr - 1)))
        return fail(IPE_ELIMIT, "head_dim %d: %d-element chunks per row must be a power of two in 2 .. 32", head_dim, ec);
    if (rot_dim < 2 || rot_dim % 2 || rot_dim > head_dim)
        return fail(IPE_EINVAL, "rot_dim %d must be even and in 2 .. head_dim", rot_dim);
    if ((rot_dim / 2) % ec) return fail(IPE_EINVAL, "rot_dim / 2 = %d must be a multiple of %d", rot_dim / 2, ec);
    if (int rc = check_half(rot_dim / 2)) return rc;
    if (inv_freq_host == nullptr) return fail(IPE_EINVAL, "inv_freq_host is NULL");
    MropeAngles a{};
    for (int j = 0; j < rot_dim / 2; ++j) {
        if (!std::isfinite(inv_freq_host[j])) return fail(IPE_EINVAL, "inv_freq[%d] is not finite", j);
        a.inv[j] = inv_freq_host[j];
    }
    if ((q_weight == nullptr) != (k_weight == nullptr)) return fail(IPE_EINVAL, "give both norm weights or neither");
    if (q_weight && (!(eps >= 0.f) || !std::isfinite(eps))) return fail(IPE_EINVAL, "eps must be finite and >= 0");
    const bool cache = slot_mapping != nullptr;
    if (!cache && (k_cache || v_cache)) return fail(IPE_EINVAL, "caches given without slot_mapping");
    if (cache && hk > 0 && k_cache == nullptr) return fail(IPE_EINVAL, "slot_mapping given without k_cache");
    if (v_cache && v == nullptr) return fail(IPE_EINVAL, "v_cache given without v");
    if (cache && (num_slots < 0 || cache_slot_stride < (long long)hk * head_dim))
        return fail(IPE_EINVAL, "num_slots must be >= 0 and cache_slot_stride >= hk * head_dim");
    if (int rc = check_qk(q, k, dtype, B, hq, hk, head_dim, q_tok_stride, k_tok_stride, "q", "k")) return rc;
    if (v_cache && hk > 0 && v_tok_stride < (long long)hk * head_dim)
        return fail(IPE_EINVAL, "v row stride %lld < heads * head_dim", (long long)v_tok_stride);
    if ((hq && (q_tok_stride % ec || !aligned(q, 16))) || (hk && (k_tok_stride % ec || !aligned(k, 16))) ||
        (v_cache && (v_tok_stride % ec || !aligned(v, 16))) ||
        (cache && (cache_slot_stride % ec || !aligned(k_cache, 16) || !aligned(v_cache, 16))) ||
        !aligned(q_weight, 16) || !aligned(k_weight, 16) || !aligned(seq_pos, 4) || !aligned(rope_deltas, 4) ||
        !aligned(slot_mapping, 8))
        return fail(IPE_EALIGN, "q, k, v, caches, weights and their strides must be 16-byte aligned");
    if (B == 0 || hq + hk == 0) return ok();
    if (int rc = check_dev(seq_pos, (size_t)B * 4, "seq_pos")) return rc;
    if (rope_deltas) {
        if (int rc = check_dev(rope_deltas, (size_t)B * 4, "rope_deltas")) return rc;
    }
    if (q_weight) {
        if (int rc = check_dev(q_weight, (size_t)head_dim * eb, "q_weight")) return rc;
        if (int rc = check_dev(k_weight, (size_t)head_dim * eb, "k_weight")) return rc;
    }
    if (cache && hk > 0) {
        if (int rc = check_dev(slot_mapping, (size_t)B * 8, "slot_mapping")) return rc;
        const size_t span = num_slots > 0 ? ((size_t)(num_slots - 1) * cache_slot_stride + (size_t)hk * head_dim) * eb : 0;
        if (int rc = check_dev(k_cache, span, "k_cache")) return rc;
        if (v_cache) {
            if (int rc = check_dev(v_cache, span, "v_cache")) return rc;
            if (int rc = check_dev(v, ((size_t)(B - 1) * v_tok_stride + (size_t)hk * head_dim) * eb, "v")) return rc;
        }
    }
    DecodeArgs d{};
    d.q = hq ? q : nullptr;
    d.k = hk ? k : nullptr;
    d.v = (v_cache && hk) ? v : nullptr;
    d.k_cache = (cache && hk) ? k_cache : nullptr;
    d.v_cache = (cache && hk) ? v_cache : nullptr;
    d.slots = (cache && hk) ? slot_mapping : nullptr;
    d.seq_pos = seq_pos;
    d.deltas = rope_deltas;
    d.q_weight = q_weight;
    d.k_weight = k_weight;
    d.B = B;
    d.q_stride = q_tok_stride;
    d.k_stride = k_tok_stride;
    d.v_stride = v_tok_stride;
    d.cache_stride = cache_slot_stride;
    d.hq = hq;
    d.hk = hk;
    d.head_dim = head_dim;
    d.half = rot_dim / 2;
    d.eps = eps;
    d.status = device_status_word();
    if (!d.status) return fail(IPE_ECUDA, "device status word unavailable");
    cudaError_t e = launch_mrope_decode(dtype == IPE_BF16, d, a, num_slots, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "mrope_decode launch");
}

static int rope_index_sizes(int64_t B, int64_t L, int n_images, int n_videos)
{
    if (B < 0 || L < 0) return fail(IPE_EINVAL, "B %lld and L %lld must be >= 0", (long long)B, (long long)L);
    if (L > (1LL << 30) || (L > 0 && B > ((1LL << 31) - 1) / L))
        return fail(IPE_ELIMIT, "B * L must stay within 2^31 - 1 and L within 2^30");
    if (n_images < 0 || n_videos < 0 || n_images > IPE_MAX_GRIDS || n_videos > IPE_MAX_GRIDS)
        return fail(IPE_ELIMIT, "n_images %d and n_videos %d must lie in 0 .. %d", n_images, n_videos, IPE_MAX_GRIDS);
    return IPE_OK;
}

size_t ipe_mrope_rope_index_workspace(int64_t B, int64_t L, int n_images, int n_videos)
{
    if (rope_index_sizes(B, L, n_images, n_videos) != IPE_OK) return 0;
    return rope_index_layout(B, L, n_images, n_videos).total;
}

int ipe_mrope_rope_index(const void *mm_token_type_ids, const void *attention_mask, int id_bytes, int64_t B, int64_t L,
                         const void *image_grid_thw, int n_images, const void *video_grid_thw, int n_videos,
                         int grid_bytes, int spatial_merge, int32_t *position_ids, int32_t *rope_deltas,
                         void *workspace, size_t workspace_bytes, void *stream)
{
    if (int rc = rope_index_sizes(B, L, n_images, n_videos)) return rc;
    if (id_bytes != 4 && id_bytes != 8) return fail(IPE_EINVAL, "id_bytes %d must be 4 or 8", id_bytes);
    if (grid_bytes != 4 && grid_bytes != 8) return fail(IPE_EINVAL, "grid_bytes %d must be 4 or 8", grid_bytes);
    if (spatial_merge < 1 || spatial_merge > 64) return fail(IPE_EINVAL, "spatial_merge %d must lie in 1 .. 64", spatial_merge);
    if (B == 0) return ok();
    const RopeIndexLayout lay = rope_index_layout(B, L, n_images, n_videos);
    if (workspace_bytes < lay.total)
        return fail(IPE_EINVAL, "workspace_bytes %zu below the %zu this call needs", workspace_bytes, lay.total);
    if (!aligned(mm_token_type_ids, id_bytes) || !aligned(attention_mask, id_bytes) ||
        !aligned(image_grid_thw, grid_bytes) || !aligned(video_grid_thw, grid_bytes) || !aligned(position_ids, 4) ||
        !aligned(rope_deltas, 4) || !aligned(workspace, 16))
        return fail(IPE_EALIGN, "ids, grids, outputs and workspace must be aligned to their element (workspace: 16 bytes)");
    const size_t slots = (size_t)B * (size_t)L;
    if (slots > 0) {
        if (int rc = check_dev(mm_token_type_ids, slots * id_bytes, "mm_token_type_ids")) return rc;
        if (attention_mask) {
            if (int rc = check_dev(attention_mask, slots * id_bytes, "attention_mask")) return rc;
        }
        if (int rc = check_dev(position_ids, 3 * slots * 4, "position_ids")) return rc;
    }
    if (int rc = check_dev(rope_deltas, (size_t)B * 4, "rope_deltas")) return rc;
    if (n_images > 0) {
        if (int rc = check_dev(image_grid_thw, (size_t)n_images * 3 * grid_bytes, "image_grid_thw")) return rc;
    }
    if (n_videos > 0) {
        if (int rc = check_dev(video_grid_thw, (size_t)n_videos * 3 * grid_bytes, "video_grid_thw")) return rc;
    }
    if (int rc = check_dev(workspace, lay.total, "workspace")) return rc;
    char *w = static_cast<char *>(workspace);
    RopeIndexArgs a{};
    a.types = mm_token_type_ids;
    a.mask = attention_mask;
    a.img_grid = image_grid_thw;
    a.vid_grid = video_grid_thw;
    a.id_bytes = id_bytes;
    a.grid_bytes = grid_bytes;
    a.B = B;
    a.L = L;
    a.tiles_per_row = (int)((L + kRiTile - 1) / kRiTile);
    a.n_img = n_images;
    a.n_vid = n_videos;
    a.merge = spatial_merge;
    a.pos = position_ids;
    a.deltas = rope_deltas;
    size_t off = 0;
    auto section = [&](size_t bytes) {
        char *p = w + off;
        off += bytes;
        return p;
    };
    a.agg = section(lay.agg);
    a.state = section(lay.state);
    a.flags = reinterpret_cast<unsigned *>(section(lay.flags));
    a.sample = section(lay.sample);
    a.ticket = reinterpret_cast<unsigned *>(section(lay.ticket));
    a.img_adv = reinterpret_cast<long long *>(section(lay.img_adv));
    a.vid_slices = reinterpret_cast<long long *>(section(lay.vid_slices));
    a.vid_adv = reinterpret_cast<long long *>(section(lay.vid_adv));
    a.wait_limit = debug_wait_limit();
    a.skip_tile = debug_skip_tile();
    a.status = device_status_word();
    if (!a.status) return fail(IPE_ECUDA, "device status word unavailable");
    cudaError_t e = launch_rope_index(a, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "rope_index launch");
}

int ipe_vis_interp_plan(const int32_t *grid_thw_host, int n_images, int merge, int grid_side, int32_t *idx4,
                        float *w4, int32_t *rowcol, void *stream)
{
    VisDesc<1024> &d = *desc_buffer();
    if (int rc = build_vis_desc(grid_thw_host, n_images, merge, grid_side, d)) return rc;
    const long long N = d.n_patch;
    if (N == 0) return ok();
    if (!aligned(idx4, 4) || !aligned(w4, 4) || !aligned(rowcol, 4)) return fail(IPE_EALIGN, "outputs not 4-byte aligned");
    if (idx4) {
        if (int rc = check_dev(idx4, (size_t)4 * N * 4, "idx4")) return rc;
    }
    if (w4) {
        if (int rc = check_dev(w4, (size_t)4 * N * 4, "w4")) return rc;
    }
    if (rowcol) {
        if (int rc = check_dev(rowcol, (size_t)2 * N * 4, "rowcol")) return rc;
    }
    cudaError_t e = launch_vis_plan(d, idx4, w4, rowcol, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "vis_interp_plan launch");
}

static int interp_args(const void *table, ipe_dtype dtype, int grid_side, int hidden, void *out,
                       const VisDesc<1024> &d, InterpArgs &ia)
{
    if (int rc = check_dtype(dtype)) return rc;
    if (hidden <= 0 || hidden % 4) return fail(IPE_EINVAL, "hidden %d must be a positive multiple of 4", hidden);
    const size_t smem = interp_smem_bytes(dtype == IPE_BF16, d.merge, grid_side);
    if (smem > 200 * 1024)
        return fail(IPE_ELIMIT, "merge %d x grid_side %d needs %zu bytes of shared memory per block", d.merge,
                    grid_side, smem);
    const int eb = elem_bytes(dtype);
    if (!aligned(table, 4 * eb) || !aligned(out, 4 * eb))
        return fail(IPE_EALIGN, "table / out must be aligned to %d bytes", 4 * eb);
    if (int rc = check_dev(table, (size_t)grid_side * grid_side * hidden * eb, "table")) return rc;
    if (int rc = check_dev(out, (size_t)d.n_patch * hidden * eb, "out")) return rc;
    const int cs = 128 / eb;
    ia.table = table;
    ia.out = out;
    ia.hidden = hidden;
    ia.n_slices = (hidden + cs - 1) / cs;
    if (ia.n_slices > 65535)   // slices are the second grid dimension
        return fail(IPE_ELIMIT, "hidden %d exceeds %d channels", hidden, 65535 * cs);
    return IPE_OK;
}

int ipe_vis_pos_interp(const void *table, ipe_dtype dtype, int grid_side, int hidden, const int32_t *grid_thw_host,
                       int n_images, int merge, void *out, void *stream)
{
    VisDesc<1024> &d = *desc_buffer();
    if (int rc = build_vis_desc(grid_thw_host, n_images, merge, grid_side, d)) return rc;
    if (d.n_patch == 0) return check_dtype(dtype) ? IPE_EINVAL : ok();
    InterpArgs ia;
    if (int rc = interp_args(table, dtype, grid_side, hidden, out, d, ia)) return rc;
    cudaError_t e = launch_vis_interp(dtype == IPE_BF16, d, ia, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "vis_pos_interp launch");
}

int ipe_vis_pos_interp_hf(const void *table, ipe_dtype dtype, int grid_side, int hidden, const int32_t *grid_thw_host,
                          int n_images, int merge, void *out, void *stream)
{
    VisDesc<1024> &d = *desc_buffer();
    if (int rc = build_vis_desc(grid_thw_host, n_images, merge, grid_side, d)) return rc;
    if (d.n_patch == 0) return check_dtype(dtype) ? IPE_EINVAL : ok();
    if (int rc = check_dtype(dtype)) return rc;
    const int ec = 16 / elem_bytes(dtype);
    if (hidden <= 0 || hidden % ec) return fail(IPE_EINVAL, "hidden %d must be a positive multiple of %d", hidden, ec);
    if (!aligned(table, 16) || !aligned(out, 16)) return fail(IPE_EALIGN, "table / out must be 16-byte aligned");
    InterpArgs ia;
    if (int rc = interp_args(table, dtype, grid_side, hidden, out, d, ia)) return rc;
    cudaError_t e = launch_vis_interp_hf(dtype == IPE_BF16, d, ia, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "vis_pos_interp_hf launch");
}

static int vis_rot_args(void *q, void *k, ipe_dtype dtype, int64_t n_patch, int heads, int head_dim,
                        int64_t q_stride, int64_t k_stride, const VisDesc<1024> &d, RotArgs &r)
{
    if (int rc = check_dtype(dtype)) return rc;
    if (n_patch != d.n_patch)
        return fail(IPE_EINVAL, "n_patch %lld != sum t h w of grid_thw = %lld", (long long)n_patch, d.n_patch);
    if (heads < 1) return fail(IPE_EINVAL, "heads %d must be >= 1", heads);
    if (q == nullptr) return fail(IPE_EINVAL, "q is NULL");
    const int hk = k ? heads : 0;
    if (int rc = check_qk(q, k, dtype, n_patch, heads, hk, head_dim, q_stride, k ? k_stride : 0, "q", "k")) return rc;
    r = RotArgs{};
    r.q = q;
    r.k = k;
    r.rows = n_patch;
    r.q_stride = q_stride;
    r.k_stride = k ? k_stride : 0;
    r.hq = heads;
    r.hk = hk;
    r.head_dim = head_dim;
    r.half = head_dim / 2;
    return IPE_OK;
}

int ipe_vis_rope2d(void *q, void *k, ipe_dtype dtype, int64_t n_patch, int heads, int head_dim, int64_t q_stride,
                   int64_t k_stride, const int32_t *grid_thw_host, int n_images, int merge, double theta, void *stream)
{
    VisDesc<1024> &d = *desc_buffer();
    if (int rc = build_vis_desc(grid_thw_host, n_images, merge, 1, d)) return rc;
    VisAngleFreqs f;
    if (int rc = vis_freqs(head_dim, theta, f)) return rc;
    if (n_patch == 0 && d.n_patch == 0) return check_dtype(dtype) ? IPE_EINVAL : ok();
    RotArgs r;
    if (int rc = vis_rot_args(q, k, dtype, n_patch, heads, head_dim, q_stride, k_stride, d, r)) return rc;
    cudaError_t e = launch_vis_rope(dtype == IPE_BF16, d, r, f, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "vis_rope2d launch");
}

// A second stream per device for work that overlaps the caller's: created on
// first use, with a ring of events (a wait refers to the record made before
// it, so the ring may wrap).
struct AuxStream {
    bool ready = false;
    cudaStream_t s = nullptr;
    cudaEvent_t ring[64] = {};
    unsigned next = 0;
};

static std::mutex g_aux_mutex;
static AuxStream g_aux[64];

static int aux_stream(AuxStream **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(IPE_ELIMIT, "device index beyond 64");
    AuxStream &a = g_aux[dev];
    if (!a.ready) {
        if ((e = cudaStreamCreateWithFlags(&a.s, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreate");
        for (cudaEvent_t &ev : a.ring)
            if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(e, "cudaEventCreate");
        a.ready = true;
    }
    *out = &a;
    return IPE_OK;
}

int ipe_vis_pos_interp_rope2d(const void *table, int grid_side, int hidden, void *out, void *q, void *k, int heads,
                              int head_dim, int64_t q_stride, int64_t k_stride, double theta, ipe_dtype dtype,
                              const int32_t *grid_thw_host, int n_images, int merge, void *stream)
{
    VisDesc<1024> &d = *desc_buffer();
    if (int rc = build_vis_desc(grid_thw_host, n_images, merge, grid_side, d)) return rc;
    VisAngleFreqs f;
    if (int rc = vis_freqs(head_dim, theta, f)) return rc;
    if (d.n_patch == 0) return check_dtype(dtype) ? IPE_EINVAL : ok();
    InterpArgs ia;
    if (int rc = interp_args(table, dtype, grid_side, hidden, out, d, ia)) return rc;
    RotArgs r;
    if (int rc = vis_rot_args(q, k, dtype, d.n_patch, heads, head_dim, q_stride, k_stride, d, r)) return rc;
    // The rotation (memory-bound) runs on `stream` and the interpolation
    // (issue-bound on single frames) on a second stream; the two kernels'
    // blocks share the SMs, and `stream` waits for both.  The rotation goes
    // first, its blocks sized to leave room for two interpolation blocks on
    // every SM when a two-stage ring still fits in what remains (else its
    // usual ring).  Measured on B200: the 16 x 64 x 64 video 134.2 -> 130.0
    // us; a batch of 8 single images (two-slice interpolation blocks of 53
    // KB) keeps the usual ring.
    const cudaStream_t s = (cudaStream_t)stream;
    std::lock_guard<std::mutex> lock(g_aux_mutex);
    AuxStream *aux = nullptr;
    if (int rc = aux_stream(&aux)) return rc;
    cudaEvent_t fork = aux->ring[aux->next++ % 64], join = aux->ring[aux->next++ % 64];
    const bool bf16 = dtype == IPE_BF16;
    // shared memory of an SM (228 KB on B200) and the 1 KB the runtime
    // reserves per block
    int dev = 0, per_sm = 0, reserve = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserve, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
        per_sm = reserve = 0;
    const size_t ib = vis_interp_block_smem(bf16, d, ia) + (size_t)reserve;
    const size_t budget = 2 * ib + reserve < (size_t)per_sm ? ((size_t)per_sm - 2 * ib) / 2 - reserve : 0;
    cudaError_t e;
    if ((e = cudaEventRecord(fork, s)) != cudaSuccess) return cuda_fail(e, "vis_pos_interp_rope2d fork");
    if ((e = launch_vis_rope(bf16, d, r, f, s, budget)) != cudaSuccess)
        return cuda_fail(e, "vis_pos_interp_rope2d rotation launch");
    if ((e = cudaStreamWaitEvent(aux->s, fork, 0)) != cudaSuccess) return cuda_fail(e, "vis_pos_interp_rope2d fork");
    if ((e = launch_vis_interp(bf16, d, ia, aux->s)) != cudaSuccess)
        return cuda_fail(e, "vis_pos_interp_rope2d interpolation launch");
    if ((e = cudaEventRecord(join, aux->s)) != cudaSuccess) return cuda_fail(e, "vis_pos_interp_rope2d join");
    if ((e = cudaStreamWaitEvent(s, join, 0)) != cudaSuccess) return cuda_fail(e, "vis_pos_interp_rope2d join");
    return ok();
}

}  // extern "C"
