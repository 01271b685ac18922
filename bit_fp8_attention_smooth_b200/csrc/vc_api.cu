// vc_api.cu -- the extern "C" entry points declared in include/vc_attention.h:
// argument validation, workspace layout, TMA tensor maps and kernel launches.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "vc_launch.cuh"



namespace {

constexpr int64_t kDefaultWaitNs = 2000000000LL;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    // offsets in bytes from the workspace base
    size_t status;
    size_t labels, c_hi, c_lo, cnorm, cent64, vnorm2, ties, tie_count, sums, cstart, ccount, hist, offs, state, vamax;  // prep region
    size_t qfp8, sq;                                                      // attention region (aliases prep)
    size_t prep_end, attn_end, total;
};

WsLayout ws_layout(const vc_shape& s, const vc_params& p) {
    const size_t BH = (size_t)s.B * s.H, N = (size_t)s.N, D = (size_t)s.d, C = (size_t)p.C;
    const size_t nblk = (N + 127) / 128;
    const size_t Cp = (C + 15) & ~size_t(15);
    WsLayout w{};
    w.status = 0;
    size_t o = 256;
    const size_t region = o;
    w.labels = o; o = align256(o + 4 * BH * N);
    w.c_hi = o; o = align256(o + 2 * BH * Cp * D);
    w.c_lo = o; o = align256(o + 2 * BH * Cp * D);
    w.cnorm = o; o = align256(o + 4 * BH * Cp);
    w.cent64 = o; o = align256(o + 8 * BH * C * D);
    w.vnorm2 = o; o = align256(o + 4 * BH * N);
    w.ties = o; o = align256(o + sizeof(vc::KmTie) * BH * N);
    w.tie_count = o; o = align256(o + (2 + 2 * vc::kKmTieRegions) * sizeof(int));  // + km_pass's regions
    w.sums = o; o = align256(o + 8 * BH * C * D);
    w.cstart = o; o = align256(o + 4 * BH * C);
    w.ccount = o; o = align256(o + 4 * BH * C);
    w.hist = o; o = align256(o + 4 * BH * C * nblk);
    w.offs = o; o = align256(o + 4 * BH * C * nblk);
    w.state = o; o = align256(o + 16 * BH);
    w.vamax = o; o = align256(o + 4 * BH * D);
    w.prep_end = o;
    o = region;
    w.qfp8 = o; o = align256(o + BH * N * D);
    w.sq = o; o = align256(o + 4 * BH * N);
    w.attn_end = o;
    w.total = w.prep_end > w.attn_end ? w.prep_end : w.attn_end;
    return w;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

vc_status check_shape_params(const vc_shape* s, const vc_params* p) {
    if (!s || !p) return VC_ERR_INVALID_ARG;
    if (s->B < 1 || s->H < 1 || s->N < 1 || (int64_t)s->B * s->H > 65535 || s->N > (1 << 24))
        return VC_ERR_INVALID_ARG;
    if (s->d != 64 && s->d != 128) return VC_ERR_UNSUPPORTED;
    if (p->block != 64 && p->block != 128) return VC_ERR_UNSUPPORTED;
    if (p->resid_fmt != 0 && p->resid_fmt != 1) return VC_ERR_INVALID_ARG;
    if (p->resid_fmt == 1 && p->block != 128) return VC_ERR_UNSUPPORTED;  // the 4-bit path: block 128
    if (p->smooth < 0 || p->smooth > 2) return VC_ERR_INVALID_ARG;
    if (p->beta < 0 || p->beta > 70) return VC_ERR_INVALID_ARG;
    if (p->wait_limit_ns < 0) return VC_ERR_INVALID_ARG;
    if (p->smooth == 1) {
        if (p->C < 1 || p->C > 256 || p->C > s->N) return VC_ERR_INVALID_ARG;
        if (p->iters < 1 || p->iters > 64) return VC_ERR_INVALID_ARG;
    }
    return VC_OK;
}

vc_status check_prep_ptrs(const vc_prep* pr, const vc_params* p, bool need_labels) {
    if (!pr) return VC_ERR_INVALID_ARG;
    if (p->resid_fmt == 1 && !aligned16(pr->v_bscale)) return VC_ERR_INVALID_ARG;
    if (!aligned16(pr->perm) || !aligned16(pr->k_fp8) || !aligned16(pr->k_scale) || !aligned16(pr->vt_fp8) ||
        !aligned16(pr->v_mean) || !aligned16(pr->v_scale))
        return VC_ERR_INVALID_ARG;
    if (need_labels && !aligned16(pr->labels)) return VC_ERR_INVALID_ARG;
    if (pr->labels && !aligned16(pr->labels)) return VC_ERR_INVALID_ARG;
    return VC_OK;
}

vc_status check_device() {
    static std::mutex mu;
    static int ok_dev[64] = {0};  // 0 unknown, 1 sm_100, -1 other
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return VC_ERR_CUDA;
    std::lock_guard<std::mutex> g(mu);
    if (ok_dev[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return VC_ERR_CUDA;
        ok_dev[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    return ok_dev[dev] == 1 ? VC_OK : VC_ERR_UNSUPPORTED;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

vc_status prepare_impl(const void* K, const void* V, const vc_shape& s, const vc_params& p, const vc_prep& out,
                       uint8_t* ws, const WsLayout& L, cudaStream_t stream) {
    vc::PrepLaunch pl{};
    pl.K = static_cast<const __nv_bfloat16*>(K);
    pl.V = static_cast<const __nv_bfloat16*>(V);
    pl.BH = s.B * s.H;
    pl.N = s.N;
    pl.D = s.d;
    pl.C = p.smooth == 1 ? p.C : 1;
    pl.iters = p.iters;
    pl.BK = p.block;
    pl.smooth = p.smooth;
    pl.resid_fmt = p.resid_fmt;
    pl.perm = out.perm;
    pl.k_fp8 = out.k_fp8;
    pl.k_scale = out.k_scale;
    pl.vt_fp8 = out.vt_fp8;
    pl.v_mean = out.v_mean;
    pl.v_scale = out.v_scale;
    pl.v_bscale = out.v_bscale;
    pl.labels = out.labels ? out.labels : reinterpret_cast<int32_t*>(ws + L.labels);
    pl.c_hi = reinterpret_cast<__nv_bfloat16*>(ws + L.c_hi);
    pl.c_lo = reinterpret_cast<__nv_bfloat16*>(ws + L.c_lo);
    pl.cnorm = reinterpret_cast<float*>(ws + L.cnorm);
    pl.cent64 = reinterpret_cast<double*>(ws + L.cent64);
    pl.vnorm2 = reinterpret_cast<float*>(ws + L.vnorm2);
    pl.ties = reinterpret_cast<vc::KmTie*>(ws + L.ties);
    pl.tie_count = reinterpret_cast<int*>(ws + L.tie_count);
    pl.sums = reinterpret_cast<double*>(ws + L.sums);
    pl.ctl.status = reinterpret_cast<int*>(ws + L.status);
    pl.ctl.limit_ns = p.wait_limit_ns > 0 ? p.wait_limit_ns : kDefaultWaitNs;
    pl.cstart = reinterpret_cast<int32_t*>(ws + L.cstart);
    pl.ccount = reinterpret_cast<int32_t*>(ws + L.ccount);
    pl.hist = reinterpret_cast<int32_t*>(ws + L.hist);
    pl.offs = reinterpret_cast<int32_t*>(ws + L.offs);
    pl.state = reinterpret_cast<vc::KmState*>(ws + L.state);
    pl.vamax = reinterpret_cast<uint32_t*>(ws + L.vamax);
    return vc::launch_prep(pl, stream) == cudaSuccess ? VC_OK : VC_ERR_CUDA;
}

vc_status attn_impl(const void* Q, const vc_prep& pr, const vc_shape& s, const vc_params& p, void* O, uint8_t* ws,
                    const WsLayout& L, cudaStream_t stream, const uint8_t* tile_mask = nullptr);
vc_status attn_impl(const void* Q, const vc_prep& pr, const vc_shape& s, const vc_params& p, void* O, uint8_t* ws,
                    const WsLayout& L, cudaStream_t stream, const uint8_t* tile_mask) {
    const int BH = s.B * s.H, N = s.N, D = s.d, BK = p.block;
    const int T = (N + BK - 1) / BK;
    const uint64_t Tp = (uint64_t)T * BK;
    uint8_t* qfp8 = ws + L.qfp8;
    float* sq = reinterpret_cast<float*>(ws + L.sq);
    if (vc::launch_quant_q(static_cast<const __nv_bfloat16*>(Q), qfp8, sq, (int64_t)BH * N, D, stream) != cudaSuccess)
        return VC_ERR_CUDA;
    CUtensorMap tk, tv;
    // V^T tiles: BK codes a channel row, bytes (E4M3) or two codes a byte (E2M1)
    const uint64_t vrow = p.resid_fmt == 1 ? Tp / 2 : Tp;
    const uint32_t vbox = p.resid_fmt == 1 ? BK / 2 : BK;
    if (!vc::make_tmap_3d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pr.k_fp8, D, Tp, BH, D, BK) ||
        !vc::make_tmap_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pr.vt_fp8, vrow, D, BH, vbox, D))
        return VC_ERR_CUDA;
    vc::AttnArgs a{};
    a.q_fp8 = qfp8;
    a.sq = sq;
    a.k_scale = pr.k_scale;
    a.v_mean = pr.v_mean;
    a.v_scale = pr.v_scale;
    a.v_bscale = pr.v_bscale;
    a.tile_mask = tile_mask;
    a.out = static_cast<__nv_bfloat16*>(O);
    a.N = N;
    a.T = T;
    a.kappa = (float)(8.0 * 1.4426950408889634074 / sqrt((double)D));
    a.beta = p.beta;
    a.ctl.status = reinterpret_cast<int*>(ws + L.status);
    a.ctl.limit_ns = p.wait_limit_ns > 0 ? p.wait_limit_ns : kDefaultWaitNs;
    const cudaError_t e = p.resid_fmt == 1 ? vc::launch_attn4(D, tk, tv, a, BH, stream)
                                           : vc::launch_attn(D, BK, tk, tv, a, BH, stream);
    return e == cudaSuccess ? VC_OK : VC_ERR_CUDA;
}

}  // namespace

namespace vc {
bool make_tmap_3d(CUtensorMap* m, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box1) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * elem_bytes, d1 * d0 * elem_bytes};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t elem[3] = {1, 1, 1};
    const uint32_t row = box0 * elem_bytes;
    const CUtensorMapSwizzle sw = row == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : row == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_32B;
    return fn(m, dtype, 3, const_cast<void*>(base), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace vc

// Scratch of vc_attn_fwd_noalloc: status word, quantised Q and its scales.
// In host code the symbol is only a handle; the device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[VC_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {nullptr};

vc_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return VC_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return VC_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return VC_OK;
}
}  // namespace

extern "C" {

int vc_abi_version(void) { return VC_ABI_VERSION; }

const char* vc_status_string(int status) {
    switch (status) {
        case VC_OK: return "ok";
        case VC_ERR_INVALID_ARG: return "invalid argument";
        case VC_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case VC_ERR_CUDA: return "CUDA error";
        case VC_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case VC_ERR_WORKSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

vc_status vc_prep_buffer_bytes(const vc_shape* shape, const vc_params* params, size_t* bytes) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!bytes) return VC_ERR_INVALID_ARG;
    const size_t BH = (size_t)shape->B * shape->H, N = shape->N, D = shape->d;
    const size_t T = (N + params->block - 1) / params->block, Tp = T * params->block;
    bytes[0] = 4 * BH * N;   // perm
    bytes[1] = 4 * BH * N;   // labels
    bytes[2] = BH * Tp * D;  // k_fp8
    bytes[3] = 4 * BH * T;   // k_scale
    const bool fp4 = params->resid_fmt == 1;
    bytes[4] = fp4 ? BH * D * Tp / 2 : BH * D * Tp;  // vt_fp8 (E2M1: two codes a byte)
    bytes[5] = 4 * BH * T * D;  // v_mean
    bytes[6] = 4 * BH * D;   // v_scale
    bytes[7] = fp4 ? BH * T * D * (params->block / 16) : 0;  // v_bscale
    return VC_OK;
}

vc_status vc_workspace_bytes(const vc_shape* shape, const vc_params* params, size_t* bytes) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!bytes) return VC_ERR_INVALID_ARG;
    *bytes = ws_layout(*shape, *params).total;
    return VC_OK;
}

vc_status vc_smooth_prepare(const void* K, const void* V, const vc_shape* shape, const vc_params* params,
                            const vc_prep* out, void* workspace, size_t workspace_bytes, void* stream) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!aligned16(K) || !aligned16(V) || !aligned16(workspace)) return VC_ERR_INVALID_ARG;
    if ((st = check_prep_ptrs(out, params, false)) != VC_OK) return st;
    const WsLayout L = ws_layout(*shape, *params);
    if (workspace_bytes < L.total) return VC_ERR_WORKSPACE;
    if ((st = check_device()) != VC_OK) return st;
    return prepare_impl(K, V, *shape, *params, *out, static_cast<uint8_t*>(workspace), L,
                        static_cast<cudaStream_t>(stream));
}

vc_status vc_attn_fwd(const void* Q, const vc_prep* prep, const vc_shape* shape, const vc_params* params, void* O,
                      void* workspace, size_t workspace_bytes, void* stream) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!aligned16(Q) || !aligned16(O) || !aligned16(workspace)) return VC_ERR_INVALID_ARG;
    if ((st = check_prep_ptrs(prep, params, false)) != VC_OK) return st;
    const WsLayout L = ws_layout(*shape, *params);
    if (workspace_bytes < L.total) return VC_ERR_WORKSPACE;
    if ((st = check_device()) != VC_OK) return st;
    return attn_impl(Q, *prep, *shape, *params, O, static_cast<uint8_t*>(workspace), L,
                     static_cast<cudaStream_t>(stream));
}

vc_status vc_attn_fwd_masked(const void* Q, const vc_prep* prep, const vc_shape* shape, const vc_params* params,
                             const uint8_t* tile_mask, void* O, void* workspace, size_t workspace_bytes,
                             void* stream) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!aligned16(Q) || !aligned16(O) || !aligned16(workspace) || !tile_mask) return VC_ERR_INVALID_ARG;
    if (params->resid_fmt != 0) return VC_ERR_UNSUPPORTED;  // the mask is read by the 8-bit kernel only
    if ((st = check_prep_ptrs(prep, params, false)) != VC_OK) return st;
    const WsLayout L = ws_layout(*shape, *params);
    if (workspace_bytes < L.total) return VC_ERR_WORKSPACE;
    if ((st = check_device()) != VC_OK) return st;
    return attn_impl(Q, *prep, *shape, *params, O, static_cast<uint8_t*>(workspace), L,
                     static_cast<cudaStream_t>(stream), tile_mask);
}

vc_status vc_attention(const void* Q, const void* K, const void* V, const vc_shape* shape, const vc_params* params,
                       const vc_prep* scratch, void* O, void* workspace, size_t workspace_bytes, void* stream) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
        return VC_ERR_INVALID_ARG;
    if ((st = check_prep_ptrs(scratch, params, false)) != VC_OK) return st;
    const WsLayout L = ws_layout(*shape, *params);
    if (workspace_bytes < L.total) return VC_ERR_WORKSPACE;
    if ((st = check_device()) != VC_OK) return st;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = prepare_impl(K, V, *shape, *params, *scratch, ws, L, s)) != VC_OK) return st;
    return attn_impl(Q, *scratch, *shape, *params, O, ws, L, s);
}

vc_status vc_attention_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, const vc_shape* shape,
                            const vc_params* params, int groups, void* Qd, void* Kd, void* Vd, void* Od,
                            const vc_prep* scratch, void* workspace, size_t workspace_bytes, void* h2d_stream,
                            void* compute_stream, void* d2h_stream) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!Qh || !Kh || !Vh || !Oh) return VC_ERR_INVALID_ARG;
    if (!aligned16(Qd) || !aligned16(Kd) || !aligned16(Vd) || !aligned16(Od) || !aligned16(workspace))
        return VC_ERR_INVALID_ARG;
    if ((st = check_prep_ptrs(scratch, params, false)) != VC_OK) return st;
    const WsLayout L = ws_layout(*shape, *params);
    if (workspace_bytes < L.total) return VC_ERR_WORKSPACE;
    if ((st = check_device()) != VC_OK) return st;
    const int64_t BH = (int64_t)shape->B * shape->H;
    const int G = groups < 1 ? 1 : (groups > BH ? (int)BH : groups);
    const int N = shape->N, D = shape->d, BK = params->block;
    const int T = (N + BK - 1) / BK;
    const size_t row = (size_t)N * D * 2;  // bytes of one (b, h) slice of Q, K, V or O
    cudaStream_t sin = static_cast<cudaStream_t>(h2d_stream);
    cudaStream_t sc = static_cast<cudaStream_t>(compute_stream);
    cudaStream_t sout = static_cast<cudaStream_t>(d2h_stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    {   // Work of an earlier call on these streams comes first: its computation
        // before this call's copies into Qd/Kd/Vd, its copies out of Od before
        // this call writes Od.
        cudaEvent_t c_prev = nullptr, o_prev = nullptr;
        if (cudaEventCreateWithFlags(&c_prev, cudaEventDisableTiming) != cudaSuccess) return VC_ERR_CUDA;
        if (cudaEventCreateWithFlags(&o_prev, cudaEventDisableTiming) != cudaSuccess) {
            cudaEventDestroy(c_prev);
            return VC_ERR_CUDA;
        }
        const bool fine = cudaEventRecord(c_prev, sc) == cudaSuccess && cudaEventRecord(o_prev, sout) == cudaSuccess &&
                          cudaStreamWaitEvent(sin, c_prev, 0) == cudaSuccess &&
                          cudaStreamWaitEvent(sc, o_prev, 0) == cudaSuccess;
        cudaEventDestroy(c_prev);
        cudaEventDestroy(o_prev);
        if (!fine) return VC_ERR_CUDA;
    }
    auto at = [](const void* p, size_t off) { return static_cast<const uint8_t*>(p) + off; };
    auto atw = [](void* p, size_t off) { return static_cast<uint8_t*>(p) + off; };
    for (int g = 0; g < G; ++g) {
        const int64_t h0 = BH * g / G, h1 = BH * (g + 1) / G;
        const int hg = (int)(h1 - h0);
        if (hg == 0) continue;
        const vc_shape gs{1, hg, N, D};
        const size_t off = (size_t)h0 * row, bytes = (size_t)hg * row;
        vc_prep gp = *scratch;  // the group's slices of the prep buffers
        gp.perm = scratch->perm + (size_t)h0 * N;
        gp.labels = scratch->labels ? scratch->labels + (size_t)h0 * N : nullptr;
        gp.k_fp8 = scratch->k_fp8 + (size_t)h0 * T * BK * D;
        gp.k_scale = scratch->k_scale + (size_t)h0 * T;
        gp.vt_fp8 = scratch->vt_fp8 + (size_t)h0 * D * T * BK / (params->resid_fmt == 1 ? 2 : 1);
        gp.v_mean = scratch->v_mean + (size_t)h0 * T * D;
        gp.v_scale = scratch->v_scale + (size_t)h0 * D;
        gp.v_bscale = params->resid_fmt == 1 ? scratch->v_bscale + (size_t)h0 * T * D * (BK / 16) : nullptr;
        cudaEvent_t in_done = nullptr, out_ready = nullptr;
        if (cudaEventCreateWithFlags(&in_done, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&out_ready, cudaEventDisableTiming) != cudaSuccess) {
            if (in_done) cudaEventDestroy(in_done);
            return VC_ERR_CUDA;
        }
        bool fine = cudaMemcpyAsync(atw(Qd, off), at(Qh, off), bytes, cudaMemcpyHostToDevice, sin) == cudaSuccess &&
                    cudaMemcpyAsync(atw(Kd, off), at(Kh, off), bytes, cudaMemcpyHostToDevice, sin) == cudaSuccess &&
                    cudaMemcpyAsync(atw(Vd, off), at(Vh, off), bytes, cudaMemcpyHostToDevice, sin) == cudaSuccess &&
                    cudaEventRecord(in_done, sin) == cudaSuccess && cudaStreamWaitEvent(sc, in_done, 0) == cudaSuccess;
        if (fine) {
            const WsLayout GL = ws_layout(gs, *params);  // a group's layout fits in the full one
            st = prepare_impl(at(Kd, off), at(Vd, off), gs, *params, gp, ws, GL, sc);
            if (st == VC_OK) st = attn_impl(at(Qd, off), gp, gs, *params, atw(Od, off), ws, GL, sc);
            fine = st == VC_OK && cudaEventRecord(out_ready, sc) == cudaSuccess &&
                   cudaStreamWaitEvent(sout, out_ready, 0) == cudaSuccess &&
                   cudaMemcpyAsync(atw(Oh, off), at(Od, off), bytes, cudaMemcpyDeviceToHost, sout) == cudaSuccess;
        }
        cudaEventDestroy(in_done);  // released once complete
        cudaEventDestroy(out_ready);
        if (!fine) return st != VC_OK ? st : VC_ERR_CUDA;
    }
    return VC_OK;
}

vc_status vc_attn_fwd_noalloc(const void* Q, const vc_prep* prep, const vc_shape* shape, const vc_params* params,
                              void* O, void* stream) {
    vc_status st = check_shape_params(shape, params);
    if (st != VC_OK) return st;
    if (!aligned16(Q) || !aligned16(O)) return VC_ERR_INVALID_ARG;
    if ((st = check_prep_ptrs(prep, params, false)) != VC_OK) return st;
    const WsLayout L = ws_layout(*shape, *params);  // the attention region only: status, Q fp8, Q scales
    if (L.attn_end > VC_NOALLOC_SCRATCH_BYTES) return VC_ERR_WORKSPACE;
    if ((st = check_device()) != VC_OK) return st;
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != VC_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch, 0, 256, s) != cudaSuccess) return VC_ERR_CUDA;  // status word starts at 0
    return attn_impl(Q, *prep, *shape, *params, O, static_cast<uint8_t*>(scratch), L, s);
}

vc_status vc_check(void* workspace, void* stream) {
    if (!aligned16(workspace)) return VC_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return VC_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return VC_ERR_CUDA;
    if (word != 0) {
        if (cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return VC_ERR_CUDA;
        return word == VC_ERR_DEVICE_TIMEOUT ? VC_ERR_DEVICE_TIMEOUT : VC_ERR_CUDA;
    }
    return VC_OK;
}

vc_status vc_e4m3_encode(const float* x, uint8_t* out, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!x || !out))) return VC_ERR_INVALID_ARG;
    vc_status st = check_device();
    if (st != VC_OK) return st;
    return vc::launch_e4m3_encode(x, out, n, static_cast<cudaStream_t>(stream)) == cudaSuccess ? VC_OK
                                                                                                : VC_ERR_CUDA;
}

vc_status vc_quantize_q(const void* Q, uint8_t* q_fp8, float* sq, int64_t tokens, int d, void* stream) {
    if (tokens < 0) return VC_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return VC_ERR_UNSUPPORTED;
    if (tokens == 0) return VC_OK;
    if (!aligned16(Q) || !aligned16(q_fp8) || !sq || (reinterpret_cast<uintptr_t>(sq) & 3u)) return VC_ERR_INVALID_ARG;
    vc_status st = check_device();
    if (st != VC_OK) return st;
    return vc::launch_quant_q(static_cast<const __nv_bfloat16*>(Q), q_fp8, sq, tokens, d,
                              static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? VC_OK
               : VC_ERR_CUDA;
}

vc_status vc_expcast_bytes(const float* A, const float* s, const float* cb, uint8_t* out, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!A || !s || !cb || !out))) return VC_ERR_INVALID_ARG;
    vc_status st = check_device();
    if (st != VC_OK) return st;
    if (n == 0) return VC_OK;
    return vc::launch_expcast(A, s, cb, out, n, static_cast<cudaStream_t>(stream)) == cudaSuccess ? VC_OK
                                                                                                 : VC_ERR_CUDA;
}

}  // extern "C"
