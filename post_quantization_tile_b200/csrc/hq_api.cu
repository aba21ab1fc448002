// hq_api.cu -- C ABI of the HyperQuant tile codec (declarations and contracts in include/hq.h):
// argument checks, TMA tensor maps, workspace set-up and kernel launches.  No allocation, no
// synchronisation except in hq_status_read.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/hq.h"
#include "../../include/hq_test.h"
#include "hq_common.cuh"
#include "hq_decode.cuh"
#include "hq_encode.cuh"
#include "hq_launch.h"

namespace hq {

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 1;
    return n;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D map over a row-major [rows, cols] tensor; box = [box_rows][128 bytes], 128-byte swizzle,
// out-of-range rows read as zero
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int es, int box_rows)
{
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const CUtensorMapDataType dt = es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : (es == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * (cuuint64_t)es};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool valid_tile(int32_t n) { return n == 64 || n == 128 || n == 256; }

struct Geometry {
    int64_t T, C, RB, items, IB;
    int TI;
};

// tiles per block item: 128 threads, `tpt` threads per tile (encoder and decoder may differ)
bool geometry(int64_t rows, int64_t cols, int32_t n, Geometry& g, int tpt = 2)
{
    if (!valid_tile(n) || rows < 1 || cols < n || cols % n) return false;
    if (rows > (int64_t)1 << 31 || cols > (int64_t)1 << 31) return false;
    const int64_t NT = cols / n;
    g.TI = kThreads / tpt;
    g.RB = (rows + kChunkTiles - 1) / kChunkTiles;
    g.C = NT * g.RB;
    g.T = NT * rows;
    g.IB = (rows + g.TI - 1) / g.TI;
    g.items = NT * g.IB;
    return true;
}

int64_t bound_words(int64_t rows, int64_t cols, int32_t n)
{
    Geometry g;
    if (!geometry(rows, cols, n, g)) return -1;
    const int64_t lmax = n / 8 + 16 * (int64_t)n + 2 * (int64_t)n;
    const int64_t words = (g.T * lmax + 31) / 32 + g.C + 8;
    return (words + 3) & ~(int64_t)3;
}

// workspace of one encoder source: the header and one look-back slot per item
size_t ws_bytes_for_src(int64_t rows, int64_t cols, int32_t n, int src)
{
    Geometry g;
    if (!geometry(rows, cols, n, g, n == 64 ? 1 : (n == 256 ? 2 : enc_tpt(128, src)))) return 0;
    return sizeof(WsHeader) + (size_t)g.items * 8u;
}

size_t ws_bytes_for(int64_t rows, int64_t cols, int32_t n)
{
    Geometry g;
    // the encoder with the most items for this tile (the one that shares a tile the most)
    if (!geometry(rows, cols, n, g, n == 64 ? 1 : (n == 256 ? 2 : enc_tpt_max(128)))) return 0;
    return sizeof(WsHeader) + (size_t)g.items * 8u;
}

bool resolve_params(const hq_params_t* p, hq_params_t& out)
{
    if (!p || !valid_tile(p->tile) || p->lattice < HQ_Z || p->lattice > HQ_E8) return false;
    out = *p;
    if (out.step == 0.0f) {
        if (!(p->bps >= 1.0f && p->bps <= 8.0f)) return false;
        out.step = hq_step_for_rate(p->lattice, p->tile, p->bps);
    }
    return out.step >= 0.00390625f && out.step <= 64.0f && std::isfinite(out.step);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Make the device that owns `p` current for this library's CUDA runtime, so that launches and
// tensor maps follow the caller's data (callers switch devices in their own runtime).
bool use_device_of(const void* p)
{
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return false;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return false;
    return cur == attr.device || cudaSetDevice(attr.device) == cudaSuccess;
}

hq_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA; }

cudaError_t run_encode(int lattice, int n, bool kv, int src, bool count, const EncodeArgs& a, const CUtensorMap& m,
                       cudaStream_t st)
{
    switch (lattice) {
    case HQ_Z: return launch_encode_z(n, kv, src, count, a, m, st);
    case HQ_A2: return launch_encode_a2(n, kv, src, count, a, m, st);
    case HQ_D4: return launch_encode_d4(n, kv, src, count, a, m, st);
    default: return launch_encode_e8(n, kv, src, count, a, m, st);
    }
}

cudaError_t run_decode(int lattice, int n, bool kv, int dst, const DecodeArgs& a, const CUtensorMap& m, cudaStream_t st)
{
    switch (lattice) {
    case HQ_Z: return launch_decode_z(n, kv, dst, a, m, st);
    case HQ_A2: return launch_decode_a2(n, kv, dst, a, m, st);
    case HQ_D4: return launch_decode_d4(n, kv, dst, a, m, st);
    default: return launch_decode_e8(n, kv, dst, a, m, st);
    }
}

// arguments, tensor map and geometry of one encode launch (src 0/1 dense input, src 2 coefficients)
struct EncodePlan {
    hq_params_t prm;
    Geometry g;
    CUtensorMap map;
    EncodeArgs a;
    bool kv;
    int src;
};

hq_status_t plan_encode(const void* x, int src, int64_t rows, int64_t cols, const hq_params_t* p, int32_t kv,
                        int64_t kv_S, int32_t* v_out, hq_code_t* out, bool count, void* ws, size_t ws_bytes,
                        EncodePlan& pl)
{
    hq_params_t& prm = pl.prm;
    if (!resolve_params(p, prm)) return HQ_ERR_ARG;
    Geometry& g = pl.g;
    const int tpt = prm.tile == 64 ? 1 : (prm.tile == 256 ? 2 : enc_tpt(128, src));
    if (!geometry(rows, cols, prm.tile, g, tpt)) return HQ_ERR_ARG;
    if (kv < 0 || kv > 2) return HQ_ERR_ARG;
    if (kv == 1 && cols != prm.tile) return HQ_ERR_ARG;
    if (src == 1 && prm.tile == 256) return HQ_ERR_UNSUPPORTED;
    if (src == 2 && cols != prm.tile) return HQ_ERR_ARG;
    if (!x || !aligned16(x) || !ws || !aligned16(ws)) return HQ_ERR_ARG;
    if (ws_bytes < sizeof(WsHeader) + (size_t)g.items * 8u) return HQ_ERR_ARG;  // this source's items
    if (!count) {
        if (!out || !out->meta || !out->chunk_word || !out->bits || out->cap_words < 1) return HQ_ERR_ARG;
        if (src != 2 && !out->scale) return HQ_ERR_ARG;
    }
    if (bound_words(rows, cols, prm.tile) >= ((int64_t)1 << 32)) return HQ_ERR_RANGE;

    if (!use_device_of(x)) return HQ_ERR_ARG;
    const int es = src == 0 ? 2 : 4;
    if (!make_map(&pl.map, x, rows, cols, es, g.TI)) return HQ_ERR_CUDA;

    EncodeArgs& a = pl.a;
    a = EncodeArgs{};
    a.rows = rows;
    a.cols = cols;
    a.beta = prm.step;
    a.seed = prm.seed;
    hq::philox_round_keys(prm.seed, a.rk);
    a.kv_S = kv == 1 ? kv_S : 0;  // 0: dither counter words (row, tile column)
    a.items = g.items;
    a.IB = g.IB;
    a.RB = g.RB;
    a.C = g.C;
    if (!count) {
        a.scale = out->scale;
        a.meta = out->meta;
        a.chunk_word = out->chunk_word;
        a.bits = out->bits;
        a.cap_words = out->cap_words;
    }
    a.v_out = v_out;
    a.ws = static_cast<WsHeader*>(ws);
    a.states = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + sizeof(WsHeader));
    a.search = nullptr;
    a.test_silent_item = -1;
    pl.kv = kv != 0;
    pl.src = src;
    return HQ_OK;
}

// common body of the encode entry points
hq_status_t encode_common(const void* x, int src, int64_t rows, int64_t cols, const hq_params_t* p, int32_t kv,
                          int64_t kv_S, int32_t* v_out, hq_code_t* out, unsigned long long* count_out, void* ws,
                          size_t ws_bytes, void* stream, int64_t kv_s0 = 0, int64_t test_silent_item = -1)
{
    const bool count = count_out != nullptr;
    if (kv_s0 < 0 || (kv_s0 && kv != 1)) return HQ_ERR_ARG;
    EncodePlan pl;
    const hq_status_t ps = plan_encode(x, src, rows, cols, p, kv, kv_S, v_out, out, count, ws, ws_bytes, pl);
    if (ps != HQ_OK) return ps;
    pl.a.kv_s0 = kv_s0;
    pl.a.test_silent_item = test_silent_item;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t clear = count ? sizeof(WsHeader) : sizeof(WsHeader) + (size_t)pl.g.items * 8u;
    cudaError_t e = cudaMemsetAsync(ws, 0, clear, st);
    if (e != cudaSuccess) return HQ_ERR_CUDA;
    e = run_encode(pl.prm.lattice, pl.prm.tile, pl.kv, src, count, pl.a, pl.map, st);
    if (e != cudaSuccess) return HQ_ERR_CUDA;
    if (count) {
        e = cudaMemcpyAsync(count_out, &pl.a.ws->count_bits, sizeof(unsigned long long), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return HQ_ERR_CUDA;
    } else {
        out->rows = rows;
        out->cols = cols;
        out->kv_S = kv == 1 ? kv_S : 0;
        out->p = pl.prm;
        out->kv = kv;
        out->kv_s0 = kv == 1 ? kv_s0 : 0;
        out->version = HQ_FORMAT_VERSION;
    }
    return HQ_OK;
}

// ---------------- step search (exact-rate mode) ----------------
constexpr int32_t kStepBitsMin = 0x3B800000;  // 2^-8
constexpr int32_t kStepBitsMax = 0x42800000;  // 64

__global__ void rate_search_init(RateSearch* s, WsHeader* h, float probe, double target, double tol, double n)
{
    h->counter = 0u;
    h->count_bits = 0ull;
    s->probe = probe;
    s->done = 0;
    s->lo = -1;
    s->hi = -1;
    s->c_lo = 0;
    s->c_hi = 0;
    s->last_side = 0;
    s->probes = 0;
    s->best = __float_as_int(probe);
    s->c_best = 0;
    s->target = target;
    s->tol = tol;
    s->n = n;
}

// one step of the search after a count-only pass (one thread).  The arithmetic is binary64 with
// explicit roundings, so that any implementation of the same rule takes the same probes.
__global__ void rate_search_update(RateSearch* s, WsHeader* h, int32_t max_probes)
{
    if (s->done) return;
    const long long c = (long long)h->count_bits;
    h->count_bits = 0ull;  // the next pass starts from a clean header
    h->counter = 0u;
    const int32_t b = __float_as_int(s->probe);
    s->probes += 1;
    const double err = fabs(__dadd_rn((double)c, -s->target));
    if (s->probes == 1 || err < fabs(__dadd_rn((double)s->c_best, -s->target))) {
        s->best = b;
        s->c_best = c;
    }
    if (err <= s->tol) {
        s->done = 1;
        return;
    }
    int side;
    if ((double)c > s->target) {
        s->lo = b;
        s->c_lo = c;
        side = 1;
    } else {
        s->hi = b;
        s->c_hi = c;
        side = 2;
    }
    long long nb;
    if (s->lo >= 0 && s->hi >= 0) {
        const int32_t lo = s->lo, hi = s->hi;
        if (hi - lo <= 1) {
            s->done = 1;
            return;
        }
        if (side == s->last_side) {
            nb = lo + (hi - lo) / 2;
        } else {
            const double t = __ddiv_rn(__dadd_rn((double)s->c_lo, -s->target), __dadd_rn((double)s->c_lo, -(double)s->c_hi));
            nb = lo + (long long)floor(__dmul_rn(t, (double)(hi - lo)));
        }
        nb = nb < lo + 1 ? lo + 1 : (nb > hi - 1 ? hi - 1 : nb);
    } else {
        // bps above the target times 2^23 binary32 steps per doubling of the step
        const double excess = __ddiv_rn(__dadd_rn((double)c, -s->target), s->n);
        double d = floor(__dadd_rn(__dmul_rn(excess, 8388608.0), 0.5));
        d = d > 134217728.0 ? 134217728.0 : (d < -134217728.0 ? -134217728.0 : d);
        nb = (long long)b + (long long)d;
        if (nb == b) nb += side == 1 ? 1 : -1;
        nb = nb < kStepBitsMin ? kStepBitsMin : (nb > kStepBitsMax ? kStepBitsMax : nb);
        if (nb == b) {
            s->done = 1;
            return;
        }
    }
    s->last_side = side;
    if (s->probes >= max_probes) {
        s->done = 1;
        return;
    }
    s->probe = __int_as_float((int32_t)nb);
}

__global__ void rate_search_finish(const RateSearch* s, hq_rate_result_t* r)
{
    r->step = __int_as_float(s->best);
    r->probes = s->probes;
    r->payload_bits = (uint64_t)s->c_best;
}

hq_status_t step_search_common(const void* x, int src, int64_t rows, int64_t cols, const hq_params_t* p, int32_t kv,
                               int64_t kv_S, int32_t max_probes, float tol_bps, hq_rate_result_t* result, void* ws,
                               size_t ws_bytes, void* stream)
{
    if (!(tol_bps <= 1.0f)) return HQ_ERR_ARG;
    if (!(tol_bps > 0.0f)) tol_bps = 0.005f;
    if (!p || !result || !aligned16(result)) return HQ_ERR_ARG;
    if (!(p->bps >= 1.0f && p->bps <= 8.0f)) return HQ_ERR_ARG;
    if (max_probes == 0) max_probes = 16;
    if (max_probes < 1 || max_probes > 64) return HQ_ERR_ARG;
    if (ws_bytes < sizeof(WsHeader) + sizeof(RateSearch)) return HQ_ERR_ARG;
    hq_params_t q = *p;
    if (!(q.step > 0.0f)) q.step = hq_step_for_rate(q.lattice, q.tile, q.bps);
    if (!(q.step >= 0.00390625f && q.step <= 64.0f)) return HQ_ERR_ARG;
    EncodePlan pl;
    const hq_status_t ps = plan_encode(x, src, rows, cols, &q, kv, kv_S, nullptr, nullptr, true, ws, ws_bytes, pl);
    if (ps != HQ_OK) return ps;
    if (!use_device_of(result)) return HQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    RateSearch* s = reinterpret_cast<RateSearch*>(static_cast<char*>(ws) + sizeof(WsHeader));
    pl.a.search = s;
    const double n = (double)rows * (double)cols;
    const double target = (double)q.bps * n;
    const double tol = (double)tol_bps * n;
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) != cudaSuccess) return HQ_ERR_CUDA;
    rate_search_init<<<1, 1, 0, st>>>(s, pl.a.ws, q.step, target, tol, n);
    if (cudaGetLastError() != cudaSuccess) return HQ_ERR_CUDA;
    for (int i = 0; i < max_probes; ++i) {
        if (run_encode(pl.prm.lattice, pl.prm.tile, pl.kv, src, true, pl.a, pl.map, st) != cudaSuccess) return HQ_ERR_CUDA;
        rate_search_update<<<1, 1, 0, st>>>(s, pl.a.ws, max_probes);
        if (cudaGetLastError() != cudaSuccess) return HQ_ERR_CUDA;
    }
    rate_search_finish<<<1, 1, 0, st>>>(s, result);
    return cuda_status(cudaGetLastError());
}

// dst: 0 bf16, 1 fp32, 2 int8 lattice codes with group scales g_out, 3 fp32 lattice points minus the
// dither in u units (KV tiles of 128, the dense inverse rotation's input)
// arguments and tensor map of one decode launch
hq_status_t plan_decode(const hq_code_t* code, void* y, int dst, int32_t kv, float* g_out, void* ws, size_t ws_bytes,
                        DecodeArgs& a, CUtensorMap& map)
{
    if (!code || !y || !aligned16(y) || !ws || !aligned16(ws)) return HQ_ERR_ARG;
    if (code->version != HQ_FORMAT_VERSION) return HQ_ERR_ARG;
    if (kv ? code->kv != 1 : (code->kv != 0 && code->kv != 2)) return HQ_ERR_ARG;
    if (dst < 0 || dst > 3) return HQ_ERR_ARG;
    if (dst == 3 && (code->kv != 1 || code->p.tile != 128)) return HQ_ERR_UNSUPPORTED;
    if (dst == 2) {
        if (!g_out || (reinterpret_cast<uintptr_t>(g_out) & 3u)) return HQ_ERR_ARG;
        if (code->kv != 0 || code->p.lattice == HQ_A2 || code->p.tile == 64) return HQ_ERR_UNSUPPORTED;
    }
    const hq_params_t& prm = code->p;
    if (!valid_tile(prm.tile) || prm.lattice < HQ_Z || prm.lattice > HQ_E8) return HQ_ERR_ARG;
    if (!(prm.step >= 0.00390625f && prm.step <= 64.0f)) return HQ_ERR_ARG;
    Geometry g;
    if (!geometry(code->rows, code->cols, prm.tile, g, dec_tpt(prm.tile))) return HQ_ERR_ARG;
    if (!code->scale || !code->meta || !code->chunk_word || !code->bits || !aligned16(code->bits)) return HQ_ERR_ARG;
    if (ws_bytes < sizeof(WsHeader)) return HQ_ERR_ARG;
    if (!use_device_of(y)) return HQ_ERR_ARG;
    const int es = dst == 0 ? 2 : (dst == 2 ? 1 : 4);
    if (!make_map(&map, y, code->rows, code->cols, es, g.TI)) return HQ_ERR_CUDA;
    a = DecodeArgs{};
    a.g_out = g_out;
    a.rows = code->rows;
    a.cols = code->cols;
    a.beta = prm.step;
    a.seed = prm.seed;
    hq::philox_round_keys(prm.seed, a.rk);
    a.kv_S = code->kv == 1 ? code->kv_S : 0;
    a.kv_s0 = code->kv == 1 ? code->kv_s0 : 0;
    if (a.kv_s0 < 0) return HQ_ERR_ARG;
    a.items = g.items;
    a.IB = g.IB;
    a.RB = g.RB;
    a.C = g.C;
    a.scale = code->scale;
    a.meta = code->meta;
    a.chunk_word = code->chunk_word;
    a.bits = code->bits;
    a.cap_words = code->cap_words;
    a.ws = static_cast<WsHeader*>(ws);
    return HQ_OK;
}

hq_status_t decode_common(const hq_code_t* code, void* y, int dst, int32_t kv, float* g_out, void* ws,
                          size_t ws_bytes, void* stream)
{
    DecodeArgs a;
    CUtensorMap map;
    const hq_status_t ps = plan_decode(code, y, dst, kv, g_out, ws, ws_bytes, a, map);
    if (ps != HQ_OK) return ps;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) != cudaSuccess) return HQ_ERR_CUDA;
    return cuda_status(run_decode(code->p.lattice, code->p.tile, code->kv != 0, dst, a, map, st));
}

// dense-rotation KV variant: the codec's workspace, then a 256-byte status block (the rotation's
// non-finite count), then the rows x 128 fp32 coefficients between the rotation and the codec
struct DenseLayout {
    size_t status_off, buf_off, total;
};
bool dense_layout(int64_t rows, DenseLayout& d)
{
    const size_t e = ws_bytes_for(rows, 128, 128);
    if (e == 0) return false;
    d.status_off = (e + 255u) & ~(size_t)255u;
    d.buf_off = d.status_off + 256u;
    d.total = d.buf_off + (((size_t)rows * 512u + 255u) & ~(size_t)255u);
    return true;
}

}  // namespace

// shared with the other translation units of the library (hq_launch.h)
bool tensor_map_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int es, int box_rows)
{
    return make_map(m, base, rows, cols, es, box_rows);
}
bool device_of(const void* p) { return use_device_of(p); }
size_t encode_workspace_bytes(int64_t rows, int64_t cols, int32_t n, int src)
{
    return valid_tile(n) ? ws_bytes_for_src(rows, cols, n, src) : 0;
}

}  // namespace hq

using namespace hq;

extern "C" {

int64_t hq_num_tiles(int64_t rows, int64_t cols, int32_t tile)
{
    Geometry g;
    return geometry(rows, cols, tile, g) ? g.T : -1;
}

int64_t hq_num_chunks(int64_t rows, int64_t cols, int32_t tile)
{
    Geometry g;
    return geometry(rows, cols, tile, g) ? g.C : -1;
}

int64_t hq_encode_bound_words(int64_t rows, int64_t cols, const hq_params_t* p)
{
    if (!p) return -1;
    return bound_words(rows, cols, p->tile);
}

size_t hq_workspace_bytes(int64_t rows, int64_t cols, const hq_params_t* p)
{
    if (!p) return 0;
    const size_t b = ws_bytes_for(rows, cols, p->tile);
    return (b + 255u) & ~(size_t)255u;
}

float hq_step_for_rate(int32_t lattice, int32_t tile, float bps)
{
    (void)tile;
    // differential entropy of N(0,1) in bits and the cell volume / dimension of each lattice
    const double h = 0.5 * std::log2(2.0 * 3.14159265358979323846 * 2.71828182845904523536);
    double logV = 0.0;
    int d = 1;
    switch (lattice) {
    case HQ_A2: logV = std::log2(std::sqrt(3.0) / 2.0); d = 2; break;
    case HQ_D4: logV = 1.0; d = 4; break;
    case HQ_E8: logV = 0.0; d = 8; break;
    default: break;
    }
    return (float)std::exp2(h - (double)bps - logV / d);
}

hq_status_t hq_encode(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                      hq_code_t* out, void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    return encode_common(x, dtype == HQ_BF16 ? 0 : 1, rows, cols, p, 0, 0, nullptr, out, nullptr, ws, ws_bytes, stream);
}

// ---------------- several weights in one launch ----------------
static_assert(HQ_BATCH_MAX == kEncodeBatchMax, "batch size of the C ABI");

size_t hq_encode_batch_workspace_bytes(int32_t count, const hq_encode_item_t* items)
{
    if (count < 1 || count > HQ_BATCH_MAX || !items) return 0;
    size_t n = sizeof(WsHeader);
    for (int32_t i = 0; i < count; ++i) {
        hq_params_t prm;
        Geometry g;
        const int src = items[i].dtype == HQ_BF16 ? 0 : 1;
        if (!resolve_params(&items[i].p, prm)) return 0;
        const int tpt = prm.tile == 64 ? 1 : (prm.tile == 256 ? 2 : enc_tpt(128, src));
        if (!geometry(items[i].rows, items[i].cols, prm.tile, g, tpt)) return 0;
        n += (size_t)g.items * 8u;
    }
    return n;
}

// one launch over several planned encodes: item i planned by plan(i, pl); finish(i, prm) fills
// item i's code header afterwards
extern "C++" {
template <typename Plan, typename Finish>
static hq_status_t encode_batch_common(int32_t count, bool kv, int src, size_t need, void* ws, void* stream, Plan plan,
                                       Finish finish)
{
    static EncodeBatch<kEncodeBatchMax> b;  // large; filled and launched under the lock
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    b = EncodeBatch<kEncodeBatchMax>{};
    int device = -1;
    int64_t item0 = 0;
    hq_params_t prm0{};
    for (int32_t i = 0; i < count; ++i) {
        EncodePlan pl;
        const hq_status_t ps = plan(i, pl);
        if (ps != HQ_OK) return ps;
        if (i == 0) prm0 = pl.prm;
        if (pl.prm.tile != prm0.tile || pl.prm.lattice != prm0.lattice) return HQ_ERR_UNSUPPORTED;
        int cur = -1;
        if (cudaGetDevice(&cur) != cudaSuccess) return HQ_ERR_CUDA;
        if (i > 0 && cur != device) return HQ_ERR_ARG;  // one device for the whole batch
        device = cur;
        pl.a.states = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + sizeof(WsHeader)) + item0;
        b.map[i] = pl.map;
        b.arg[i] = pl.a;
        b.item0[i] = item0;
        item0 += pl.g.items;
    }
    if (kv && prm0.tile != 128) return HQ_ERR_UNSUPPORTED;
    b.item0[count] = item0;
    b.count = count;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, need, st) != cudaSuccess) return HQ_ERR_CUDA;
    cudaError_t e;
    switch (prm0.lattice) {
    case HQ_Z: e = launch_encode_batch_z(prm0.tile, kv, src, b, st); break;
    case HQ_A2: e = launch_encode_batch_a2(prm0.tile, kv, src, b, st); break;
    case HQ_D4: e = launch_encode_batch_d4(prm0.tile, kv, src, b, st); break;
    default: e = launch_encode_batch_e8(prm0.tile, kv, src, b, st); break;
    }
    if (e != cudaSuccess) return HQ_ERR_CUDA;
    for (int32_t i = 0; i < count; ++i) finish(i, prm0);
    return HQ_OK;
}
}  // extern "C++"

hq_status_t hq_encode_batch(int32_t count, const hq_encode_item_t* items, void* ws, size_t ws_bytes, void* stream)
{
    if (count < 1 || count > HQ_BATCH_MAX || !items || !ws) return HQ_ERR_ARG;
    const size_t need = hq_encode_batch_workspace_bytes(count, items);
    if (need == 0 || ws_bytes < need) return HQ_ERR_ARG;
    for (int32_t i = 0; i < count; ++i) {
        if (items[i].dtype != HQ_BF16 && items[i].dtype != HQ_F32) return HQ_ERR_ARG;
        if (items[i].dtype != items[0].dtype) return HQ_ERR_UNSUPPORTED;
    }
    const int src = items[0].dtype == HQ_BF16 ? 0 : 1;
    return encode_batch_common(
        count, false, src, need, ws, stream,
        [&](int32_t i, EncodePlan& pl) {
            const hq_encode_item_t& it = items[i];
            return plan_encode(it.x, src, it.rows, it.cols, &it.p, 0, 0, nullptr, it.out, false, ws, ws_bytes, pl);
        },
        [&](int32_t i, const hq_params_t&) {
            hq_code_t* out = items[i].out;
            out->rows = items[i].rows;
            out->cols = items[i].cols;
            out->kv_S = 0;
            resolve_params(&items[i].p, out->p);
            out->kv = 0;
            out->kv_s0 = 0;
            out->version = HQ_FORMAT_VERSION;
        });
}

size_t hq_kv_encode_batch_workspace_bytes(int32_t count, const hq_kv_item_t* items)
{
    if (count < 1 || count > HQ_BATCH_MAX || !items) return 0;
    size_t n = sizeof(WsHeader);
    for (int32_t i = 0; i < count; ++i) {
        const hq_kv_item_t& it = items[i];
        if (it.B < 1 || it.H < 1 || it.S < 1 || it.B * it.H > ((int64_t)1 << 32)) return 0;
        hq_params_t prm;
        Geometry g;
        if (!resolve_params(&it.p, prm) || it.D != prm.tile) return 0;
        const int tpt = prm.tile == 64 ? 1 : (prm.tile == 256 ? 2 : enc_tpt(128, it.dtype == HQ_BF16 ? 0 : 1));
        if (!geometry(it.B * it.H * it.S, it.D, prm.tile, g, tpt)) return 0;
        n += (size_t)g.items * 8u;
    }
    return n;
}

hq_status_t hq_kv_encode_batch(int32_t count, const hq_kv_item_t* items, void* ws, size_t ws_bytes, void* stream)
{
    if (count < 1 || count > HQ_BATCH_MAX || !items || !ws) return HQ_ERR_ARG;
    const size_t need = hq_kv_encode_batch_workspace_bytes(count, items);
    if (need == 0 || ws_bytes < need) return HQ_ERR_ARG;
    for (int32_t i = 0; i < count; ++i) {
        if (items[i].dtype != HQ_BF16 && items[i].dtype != HQ_F32) return HQ_ERR_ARG;
        if (items[i].s0 < 0) return HQ_ERR_ARG;
        if (items[i].dtype != items[0].dtype) return HQ_ERR_UNSUPPORTED;
    }
    const int src = items[0].dtype == HQ_BF16 ? 0 : 1;
    return encode_batch_common(
        count, true, src, need, ws, stream,
        [&](int32_t i, EncodePlan& pl) {
            const hq_kv_item_t& it = items[i];
            const hq_status_t ps = plan_encode(it.kv, src, it.B * it.H * it.S, it.D, &it.p, 1, it.S, nullptr, it.out,
                                               false, ws, ws_bytes, pl);
            pl.a.kv_s0 = it.s0;
            return ps;
        },
        [&](int32_t i, const hq_params_t&) {
            const hq_kv_item_t& it = items[i];
            hq_code_t* out = it.out;
            out->rows = it.B * it.H * it.S;
            out->cols = it.D;
            out->kv_S = it.S;
            resolve_params(&it.p, out->p);
            out->kv = 1;
            out->kv_s0 = it.s0;
            out->version = HQ_FORMAT_VERSION;
        });
}

hq_status_t hq_decode_batch(int32_t count, const hq_decode_item_t* items, void* ws, size_t ws_bytes, void* stream)
{
    if (count < 1 || count > HQ_BATCH_MAX || !items || !ws) return HQ_ERR_ARG;
    static DecodeBatch<kEncodeBatchMax> b;  // large; filled and launched under the lock
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    b = DecodeBatch<kEncodeBatchMax>{};
    int device = -1;
    int64_t item0 = 0;
    for (int32_t i = 0; i < count; ++i) {
        const hq_decode_item_t& it = items[i];
        if (!it.code) return HQ_ERR_ARG;
        if (it.dtype != HQ_BF16 && it.dtype != HQ_F32) return HQ_ERR_ARG;
        if (it.dtype != items[0].dtype || it.code->kv != 0 || !items[0].code ||
            it.code->p.tile != items[0].code->p.tile || it.code->p.lattice != items[0].code->p.lattice)
            return HQ_ERR_UNSUPPORTED;
        const hq_status_t ps = plan_decode(it.code, it.y, it.dtype == HQ_BF16 ? 0 : 1, 0, nullptr, ws, ws_bytes,
                                           b.arg[i], b.map[i]);
        if (ps != HQ_OK) return ps;
        int cur = -1;
        if (cudaGetDevice(&cur) != cudaSuccess) return HQ_ERR_CUDA;
        if (i > 0 && cur != device) return HQ_ERR_ARG;  // one device for the whole batch
        device = cur;
        b.item0[i] = item0;
        item0 += b.arg[i].items;
    }
    b.item0[count] = item0;
    b.count = count;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) != cudaSuccess) return HQ_ERR_CUDA;
    const int n = items[0].code->p.tile, dst = items[0].dtype == HQ_BF16 ? 0 : 1;
    cudaError_t e;
    switch (items[0].code->p.lattice) {
    case HQ_Z: e = launch_decode_batch_z(n, dst, b, st); break;
    case HQ_A2: e = launch_decode_batch_a2(n, dst, b, st); break;
    case HQ_D4: e = launch_decode_batch_d4(n, dst, b, st); break;
    default: e = launch_decode_batch_e8(n, dst, b, st); break;
    }
    return cuda_status(e);
}

hq_status_t hq_encode_dither(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                             hq_code_t* out, void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    return encode_common(x, dtype == HQ_BF16 ? 0 : 1, rows, cols, p, 2, 0, nullptr, out, nullptr, ws, ws_bytes, stream);
}

hq_status_t hq_decode(const hq_code_t* code, void* y, hq_dtype_t dtype, void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    return decode_common(code, y, dtype == HQ_BF16 ? 0 : 1, 0, nullptr, ws, ws_bytes, stream);
}

hq_status_t hq_decode_int8(const hq_code_t* code, int8_t* v_out, float* g_out, void* ws, size_t ws_bytes, void* stream)
{
    return decode_common(code, v_out, 2, 0, g_out, ws, ws_bytes, stream);
}

hq_status_t hq_kv_encode(const void* kv, hq_dtype_t dtype, int64_t B, int64_t H, int64_t S, int64_t D,
                         const hq_params_t* p, hq_code_t* out, void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (B < 1 || H < 1 || S < 1 || !p || D != p->tile) return HQ_ERR_ARG;
    if (B * H > ((int64_t)1 << 32)) return HQ_ERR_ARG;
    return encode_common(kv, dtype == HQ_BF16 ? 0 : 1, B * H * S, D, p, 1, S, nullptr, out, nullptr, ws, ws_bytes,
                         stream);
}

hq_status_t hq_kv_encode_at(const void* kv, hq_dtype_t dtype, int64_t B, int64_t H, int64_t S, int64_t D, int64_t s0,
                            const hq_params_t* p, hq_code_t* out, void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (B < 1 || H < 1 || S < 1 || s0 < 0 || !p || D != p->tile) return HQ_ERR_ARG;
    if (B * H > ((int64_t)1 << 32)) return HQ_ERR_ARG;
    return encode_common(kv, dtype == HQ_BF16 ? 0 : 1, B * H * S, D, p, 1, S, nullptr, out, nullptr, ws, ws_bytes,
                         stream, s0);
}

hq_status_t hq_kv_decode(const hq_code_t* code, void* kv, hq_dtype_t dtype, void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    return decode_common(code, kv, dtype == HQ_BF16 ? 0 : 1, 1, nullptr, ws, ws_bytes, stream);
}

size_t hq_kv_dense_workspace_bytes(int64_t rows)
{
    DenseLayout d;
    return rows >= 1 && dense_layout(rows, d) ? d.total : 0;
}

hq_status_t hq_kv_encode_dense(const void* kv, hq_dtype_t dtype, int64_t B, int64_t H, int64_t S, int64_t D,
                               int64_t s0, const float* Q, const hq_params_t* p, hq_code_t* out, void* ws,
                               size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (B < 1 || H < 1 || S < 1 || s0 < 0 || !p || !Q || !out || D != p->tile) return HQ_ERR_ARG;
    if (D != 128) return HQ_ERR_UNSUPPORTED;
    if (B * H > ((int64_t)1 << 32) || B * H * S > ((int64_t)1 << 31)) return HQ_ERR_ARG;
    hq_params_t prm;
    if (!resolve_params(p, prm)) return HQ_ERR_ARG;
    const int64_t rows = B * H * S;
    DenseLayout d;
    if (!dense_layout(rows, d) || ws_bytes < d.total) return HQ_ERR_ARG;
    if (!kv || !aligned16(kv) || (reinterpret_cast<uintptr_t>(Q) & 3u) || !ws || !aligned16(ws)) return HQ_ERR_ARG;
    if (!out->scale || !out->meta || !out->chunk_word || !out->bits || out->cap_words < 1) return HQ_ERR_ARG;
    if (!use_device_of(kv)) return HQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    uint32_t* nonfinite = reinterpret_cast<uint32_t*>(w + d.status_off);
    float* u = reinterpret_cast<float*>(w + d.buf_off);
    if (cudaMemsetAsync(nonfinite, 0, sizeof(uint32_t), st) != cudaSuccess) return HQ_ERR_CUDA;
    if (launch_rotate(kv, dtype == HQ_BF16, Q, prm.step, rows, u, out->scale, nonfinite, st) != cudaSuccess)
        return HQ_ERR_CUDA;
    hq_code_t body = *out;
    body.scale = nullptr;  // the rotation wrote the scales
    const hq_status_t s = encode_common(u, 2, rows, D, &prm, 1, S, nullptr, &body, nullptr, ws, ws_bytes, stream, s0);
    if (s != HQ_OK) return s;
    if (launch_merge_nonfinite(ws, nonfinite, st) != cudaSuccess) return HQ_ERR_CUDA;
    out->rows = body.rows;
    out->cols = body.cols;
    out->kv_S = body.kv_S;
    out->p = body.p;
    out->kv = 3;
    out->kv_s0 = body.kv_s0;
    out->version = body.version;
    return HQ_OK;
}

hq_status_t hq_kv_decode_dense(const hq_code_t* code, const float* Q, void* kv, hq_dtype_t dtype, void* ws,
                               size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (!code || code->kv != 3 || !Q || (reinterpret_cast<uintptr_t>(Q) & 3u)) return HQ_ERR_ARG;
    if (!kv || !aligned16(kv) || !ws || !aligned16(ws)) return HQ_ERR_ARG;
    if (code->cols != code->p.tile || code->rows < 1) return HQ_ERR_ARG;
    if (code->p.tile != 128) return HQ_ERR_UNSUPPORTED;
    DenseLayout d;
    if (!dense_layout(code->rows, d) || ws_bytes < d.total) return HQ_ERR_ARG;
    if (!use_device_of(kv)) return HQ_ERR_ARG;
    float* pbuf = reinterpret_cast<float*>(static_cast<char*>(ws) + d.buf_off);
    hq_code_t body = *code;
    body.kv = 1;  // dither words of KV rows; the lattice points come back untransformed
    const hq_status_t s = decode_common(&body, pbuf, 3, 1, nullptr, ws, ws_bytes, stream);
    if (s != HQ_OK) return s;
    return launch_unrotate(pbuf, Q, code->scale, code->p.step, code->rows, kv, dtype == HQ_BF16, ws,
                           static_cast<cudaStream_t>(stream)) == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

hq_status_t hq_quantize_coeffs(const float* u, int64_t tiles, const hq_params_t* p, int32_t kv, int64_t kv_S,
                               int32_t* v_out, hq_code_t* out, void* ws, size_t ws_bytes, void* stream)
{
    if (!p) return HQ_ERR_ARG;
    hq_params_t q = *p;
    if (q.step == 0.0f) q.step = 1.0f;  // unused on this path (coefficients are already normalised)
    return encode_common(u, 2, tiles, p->tile, &q, kv, kv ? (kv_S > 0 ? kv_S : tiles) : 0, v_out, out, nullptr, ws,
                         ws_bytes, stream);
}

hq_status_t hq_encode_count(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                            int32_t kv, int64_t kv_S, uint64_t* bits_out, void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (!bits_out) return HQ_ERR_ARG;
    return encode_common(x, dtype == HQ_BF16 ? 0 : 1, rows, cols, p, kv, kv ? kv_S : 0, nullptr, nullptr,
                         reinterpret_cast<unsigned long long*>(bits_out), ws, ws_bytes, stream);
}

hq_status_t hq_step_search(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols, const hq_params_t* p,
                           int32_t kv, int64_t kv_S, int32_t max_probes, float tol_bps, hq_rate_result_t* result,
                           void* ws, size_t ws_bytes, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    return step_search_common(x, dtype == HQ_BF16 ? 0 : 1, rows, cols, p, kv, kv ? kv_S : 0, max_probes, tol_bps,
                              result, ws, ws_bytes, stream);
}

#ifdef HQ_TEST_HOOKS
// only in the test library (libhq_test.so): the product library does not export it
hq_status_t hq_test_encode_silent_item(const void* x, hq_dtype_t dtype, int64_t rows, int64_t cols,
                                       const hq_params_t* p, hq_code_t* out, void* ws, size_t ws_bytes,
                                       int64_t silent_item, void* stream)
{
    if (dtype != HQ_BF16 && dtype != HQ_F32) return HQ_ERR_ARG;
    if (silent_item < 1) return HQ_ERR_ARG;  // item 0 needs no look-back
    if (!p || p->lattice != HQ_E8) return HQ_ERR_UNSUPPORTED;  // the E8 kernels carry the hook
    return encode_common(x, dtype == HQ_BF16 ? 0 : 1, rows, cols, p, 0, 0, nullptr, out, nullptr, ws, ws_bytes, stream,
                         0, silent_item);
}
#endif

hq_status_t hq_status_read(const void* ws, void* stream, int64_t* detail)
{
    if (!ws) return HQ_ERR_ARG;
    if (!use_device_of(ws)) return HQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return HQ_ERR_CUDA;
    WsHeader h;
    if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return HQ_ERR_CUDA;
    const hq_status_t order[] = {HQ_ERR_TIMEOUT, HQ_ERR_CORRUPT, HQ_ERR_CAPACITY, HQ_ERR_RANGE, HQ_ERR_NONFINITE};
    for (hq_status_t s : order) {
        if (h.status & (1u << s)) {
            if (detail) *detail = s == HQ_ERR_CAPACITY ? (int64_t)h.needed : (s == HQ_ERR_NONFINITE ? (int64_t)h.nonfinite : 0);
            return s;
        }
    }
    if (detail) *detail = (int64_t)h.needed;
    return HQ_OK;
}

const char* hq_status_str(hq_status_t s)
{
    switch (s) {
    case HQ_OK: return "ok";
    case HQ_ERR_ARG: return "invalid argument";
    case HQ_ERR_UNSUPPORTED: return "unsupported combination";
    case HQ_ERR_CAPACITY: return "bitstream buffer too small";
    case HQ_ERR_NONFINITE: return "non-finite input (tile coded as zeros)";
    case HQ_ERR_CORRUPT: return "corrupt code stream";
    case HQ_ERR_TIMEOUT: return "bounded wait ran out";
    case HQ_ERR_RANGE: return "value out of range";
    case HQ_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

int32_t hq_version(void) { return HQ_FORMAT_VERSION; }

}  // extern "C"
