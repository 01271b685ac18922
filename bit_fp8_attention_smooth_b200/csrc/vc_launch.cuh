// vc_launch.cuh -- argument blocks and launchers shared by the entry points
// (vc_api.cu) and the kernels (vc_attn.cu, vc_prep.cu).
#pragma once

#include <atomic>

#include "vc_device.cuh"

namespace vc {

// Kernel attributes such as the dynamic shared-memory limit belong to one
// device: a launcher sets them once for each device it runs on (a bit per
// device, ordinals 0..63).  Two threads may both set them the first time,
// which is harmless.
struct PerDeviceOnce {
    std::atomic<uint64_t> mask{0};
    static int current() {
        int d = -1;
        return cudaGetDevice(&d) == cudaSuccess ? d : -1;
    }
    bool done(int dev) const { return dev >= 0 && dev < 64 && ((mask.load() >> dev) & 1u); }
    void mark(int dev) {
        if (dev >= 0 && dev < 64) mask.fetch_or(uint64_t(1) << dev);
    }
};

// Streaming multiprocessors of the current device, queried once per device
// (grid sizes of the grid-stride kernels scale with it).
inline int sm_count() {
    static std::atomic<int> cache[64];
    const int dev = PerDeviceOnce::current();
    if (dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load();
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n);
    }
    return n;
}

struct AttnArgs {
    const uint8_t* q_fp8;  // [BH, N, D] E4M3 Q
    const float* sq;       // [BH, N] per-token Q scale
    const float* k_scale;  // [BH, T]
    const float* v_mean;   // [BH, T, D]
    const float* v_scale;  // [BH, D]
    const uint8_t* v_bscale;  // 4-bit path: [BH, T, D, BK/16] UE4M3 block scales of the V residual
    const uint8_t* tile_mask; // block-sparse: [BH, Tq, T], nonzero keeps key tile t for query tile q; null: dense
    __nv_bfloat16* out;    // [BH, N, D]
    int N, T;
    float kappa;  // fp32(8 * log2(e) / sqrt(D))
    int beta;
    DevCtl ctl;
};

struct KmState {  // per (b, h), 16 bytes of workspace
    int chg[2];  // labels changed by pass it, in chg[it % 2]
    int done;    // the labels stopped changing: the regroup is final
    int pad;
};

// The fused k-means pass lists near ties in one region per CTA (one CTA per
// SM); the workspace holds the (start, count) pairs of this many regions.
constexpr int kKmTieRegions = 1024;

// A k-means near tie: a token whose tensor-core distances leave more than one
// cluster within the error bound; km_refine decides it in fp64.
struct KmTie {
    int32_t bh, n;       // head, token
    int32_t old, prov;   // label before this pass (-1 on the first), tensor-core label
    uint32_t mask[8];    // candidate clusters (bit k of word k / 32)
};

struct PrepLaunch {
    const __nv_bfloat16* K;
    const __nv_bfloat16* V;
    int BH, N, D, C, iters, BK, smooth;
    int resid_fmt;  // 0: E4M3 residual; 1: 4-bit (NVFP4) residual
    // outputs
    int32_t* perm;
    uint8_t* k_fp8;
    float* k_scale;
    uint8_t* vt_fp8;    // E4M3 residual, or E2M1 codes two a byte
    float* v_mean;
    float* v_scale;
    uint8_t* v_bscale;  // 4-bit path: [BH, T, D, BK/16] UE4M3 block scales
    // workspace
    int32_t* labels;
    __nv_bfloat16* c_hi;  // [BH, Cp, D] centroid high bf16 part
    __nv_bfloat16* c_lo;  // [BH, Cp, D] centroid residual bf16 part
    float* cnorm;         // [BH, Cp] squared centroid norms
    double* cent64;       // [BH, C, D] fp64 centroids (the exact near-tie decision)
    double* sums;         // [BH, C, D] fp64 member sums of the Lloyd update
    float* vnorm2;        // [BH, N] |v|^2 of every token (bounds the tensor-core distance error)
    KmTie* ties;          // [BH * N] near-tie list of the current pass
    int* tie_count;       // [2] list lengths, by pass parity
    int32_t* cstart;
    int32_t* ccount;
    int32_t* hist;
    int32_t* offs;
    KmState* state;
    uint32_t* vamax;
    DevCtl ctl;
};

// 3-D tensor map over a dense [d2][d1][d0] array of elem_bytes elements with
// box {box0, box1, 1}; the swizzle matches box0 * elem_bytes (128, 64 or 32 B).
bool make_tmap_3d(CUtensorMap* m, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box1);

cudaError_t launch_attn(int D, int BK, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int BH,
                        cudaStream_t stream);
// The 4-bit path (block 128): NVFP4 P and V residual in the PV product.
cudaError_t launch_attn4(int D, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int BH,
                         cudaStream_t stream);
cudaError_t launch_prep(const PrepLaunch& p, cudaStream_t s);
cudaError_t launch_quant_q(const __nv_bfloat16* Q, uint8_t* q_fp8, float* sq, int64_t tokens, int D,
                           cudaStream_t s);
cudaError_t launch_e4m3_encode(const float* x, uint8_t* out, int64_t n, cudaStream_t s);
cudaError_t launch_expcast(const float* A, const float* s, const float* cb, uint8_t* out, int64_t n,
                           cudaStream_t stream);

}  // namespace vc
