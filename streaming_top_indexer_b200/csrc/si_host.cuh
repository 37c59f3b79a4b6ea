// si_host.cuh -- host-side pieces shared by the C-ABI library (si_lib.cu)
// and the translation units that instantiate the select kernel, one per H_I
// (si_select_h8/16/32/64.cu, compiled in parallel): launch constants, the
// launch description, TMA descriptor encoding and the launch template.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "si.h"
#include "si_select.cuh"

namespace si_host {

constexpr int kMaxCtas = 148;                 // persistent CTAs (one per B200 SM)
constexpr size_t kHeaderBytes = 256;          // workspace header: error word + reserved
constexpr uint32_t kMaxDynSmem = 232448;      // 227 KB opt-in per block on sm_100
constexpr uint32_t kMinDynSmem = 120 * 1024;  // > half an SM: one CTA per SM, so
                                              // two CTAs never compete for TMEM

// One select-kernel launch, fully decided by the library's host code.
struct SelectLaunch {
    const void* q;
    const float* w;
    const void* kc;
    int64_t B, S, T;
    int H, D, m, k;
    int32_t* out_idx;
    float* out_score;
    float* dense;        // dense-score mode, else nullptr
    void* ws;            // workspace (its header holds the error word)
    cudaStream_t stream;
    int64_t t_lo, t_hi;  // query rows [t_lo, t_hi) of every batch
    bool smem_pool;      // candidate pools in shared memory (else gpool)
    int P;               // pool capacity per query
    int sort_e;          // unit-end row sort: 128 * sort_e keys per row, 0 = none
    uint32_t check_tiles, cut_slack;
    uint64_t timeout_ns;
    uint64_t* gpool;
    unsigned long long* trace;
};

// Defined in si_lib.cu.
si_status cuda_fail(const char* where, cudaError_t e);
int device_sms(int dev);
uint64_t timeout_ns();  // device wait limit set by si_set_timeout_ns
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
               uint64_t stride1_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw);
bool encode_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw);

// Defined in si_select_h<H>.cu: launch for that H_I and a.D.
si_status launch_select_h8(const SelectLaunch& a);
si_status launch_select_h16(const SelectLaunch& a);
si_status launch_select_h32(const SelectLaunch& a);
si_status launch_select_h64(const SelectLaunch& a);

// Tensor maps, shared-memory attribute and launch of select_kernel<H, D>.
//   q:  {d_I, S*H_I, B}, box {64, 256} (one unit's rows), 128-byte swizzle
//   kc: {d_I, T, B},     box {64, 128} (one key tile),    128-byte swizzle
//   w:  {H_I, S, B},     box {H_I, 256/H_I},              no swizzle
template <int H, int D>
si_status launch_select_t(const SelectLaunch& a) {
    using C = si::SelCfg<H, D>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SI_ERR_CUDA;
    const int sms = device_sms(dev);
    if (sms <= 0) return SI_ERR_CUDA;

    si::SelectParams p{};
    p.B = a.B;
    p.S = a.S;
    p.T = a.T;
    p.m = a.m;
    p.k = a.k;
    p.P = a.P;
    p.t_lo = a.t_lo;
    p.t_hi = a.t_hi;
    p.nblk = (a.t_hi - a.t_lo + C::QT - 1) / C::QT;
    p.units = a.B * p.nblk;
    p.out_idx = a.out_idx;
    p.out_score = a.out_score;
    p.dense = a.dense;
    p.gpool = a.gpool;
    p.err = static_cast<uint32_t*>(a.ws);
    p.sort_e = a.sort_e;
    p.check_tiles = a.check_tiles;
    p.cut_slack = a.cut_slack;
    p.timeout_ns = a.timeout_ns;
    p.trace = a.trace;

    CUtensorMap tq, tkc, tw;
    const uint64_t bf = 2;
    const uint64_t S = static_cast<uint64_t>(a.S), T = static_cast<uint64_t>(a.T), B = static_cast<uint64_t>(a.B);
    if (!encode_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, D, S * H, B, D * bf, S * H * D * bf, 64, C::N,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return SI_ERR_CUDA;
    if (!encode_3d(&tkc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.kc, D, T, B, D * bf, T * D * bf, 64, C::BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return SI_ERR_CUDA;
    if (!encode_3d(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.w, H, S, B, H * 4ull, S * H * 4ull, H, C::QT,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
        return SI_ERR_CUDA;

    uint32_t smem = C::dyn_bytes(a.smem_pool, p.P);
    if (smem < kMinDynSmem) smem = kMinDynSmem;
    if (smem + C::STATIC_BYTES > kMaxDynSmem) return SI_ERR_UNSUPPORTED;
    auto kern = a.smem_pool ? si::select_kernel<H, D, true> : si::select_kernel<H, D, false>;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SI_ERR_CUDA;
    if (fa.sharedSizeBytes > C::STATIC_BYTES) return SI_ERR_UNSUPPORTED;  // build drifted past the bound
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail("select kernel shared-memory attribute", e);
    int64_t grid = sms < kMaxCtas ? sms : kMaxCtas;
    if (grid > p.units) grid = p.units;
    kern<<<static_cast<unsigned>(grid), C::THREADS, smem, a.stream>>>(tq, tkc, tw, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? SI_OK : cuda_fail("select kernel launch", e);
}

}  // namespace si_host
