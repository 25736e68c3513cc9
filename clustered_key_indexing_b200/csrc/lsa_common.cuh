// lsa_common.cuh -- shared device helpers of the LSA CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "lsa.h"

namespace lsa {

// Geometry fixed by the LSA pages (essay "《卡片柜》", ch. 2): 64-d latent,
// 4 keys pooled per unit, 512-key cluster blocks (128 units) split into
// buckets of mean 8 keys (64 per block) and at most 16 keys (4 units).
constexpr int kD = 128;            // d_head
constexpr int kDL = 64;            // d_latent
constexpr int kPool = 4;
constexpr int kBlockKeys = 512;
constexpr int kUnitsPerBlock = 128;
constexpr int kBucketsPerBlock = 64;
constexpr int kMaxUnits = 4;
constexpr int kIMax = 2147483647;

// Device-side error word (one per device; the library is one translation
// unit, lsa_lib.cu): kernels that detect an
// inconsistency store a code here instead of trapping; the host reads it
// with lsa_check_device_error().
__device__ int g_lsa_device_error = 0;

enum DeviceError : int {
    kErrNone = 0,
    kErrWardInfeasible = 1,   // no eligible pair before the target count
    kErrSelectOverflow = 2,   // candidate list exceeded its capacity
    kErrIndexRange = 3,       // an index list entry was >= T
    kErrTcTimeout = 4,        // a tensor-core pipeline wait ran out (mbarrier never completed)
};

// Rows of the flat search that took the exact fallback (diagnostics).
__device__ unsigned long long g_lsa_fallback_rows = 0ull;

__device__ __forceinline__ void raise_device_error(int code) {
    atomicCAS(&g_lsa_device_error, 0, code);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
    return __uint_as_float(((uint32_t)h) << 16);
}

__device__ __forceinline__ double bf16_to_f64(uint16_t h) {
    return (double)bf16_to_f32(h);
}

// Round a double directly to bf16 (8 significant bits), ties to even: add
// half an ulp minus one (plus the kept lsb) to the bit pattern and truncate
// the 45 dropped mantissa bits; tiny magnitudes use bf16's fixed subnormal
// spacing 2^-133.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
    if (isnan(x)) return 0x7FC0;
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    const double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    const unsigned long long b = (unsigned long long)__double_as_longlong(a);
    const int e = (int)(b >> 52) - 1023;
    double y;
    if (e >= -126) {
        unsigned long long r = b + ((1ull << 44) - 1ull) + ((b >> 45) & 1ull);
        r &= ~((1ull << 45) - 1ull);
        y = __longlong_as_double((long long)r);
    } else {
        y = rint(a * 0x1p133) * 0x1p-133;  // exact power-of-two scalings
    }
    const float f = __double2float_rn(y);  // exact, or inf past the bf16 range
    return (uint16_t)(sign | (uint16_t)(__float_as_uint(f) >> 16));
}

// OCP FP8 E4M3 ("fn": bias 7, 3 mantissa bits, no infinities, largest
// finite 448, exponent field 0 = subnormals m * 2^-9).  Round a double to
// the nearest code, ties to the even mantissa, saturating at +-448: normal
// magnitudes keep the top 3 of the 52 mantissa bits (a carry out of them
// moves to the next exponent), magnitudes below 2^-6 are the integer
// nearest a * 2^9 (0 .. 8, where 8 is the smallest normal, code 0x08).
__device__ __forceinline__ uint8_t f64_to_e4m3_rne(double x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0;
    const double a = fabs(x);
    if (a == 0.0) return sign;
    const unsigned long long b = (unsigned long long)__double_as_longlong(a);
    const int e = (int)(b >> 52) - 1023;  // a in [2^e, 2^(e+1))
    if (e >= -6) {
        if (e > 8) return (uint8_t)(sign | 0x7E);
        const unsigned long long mant = b & ((1ull << 52) - 1ull);
        uint32_t q = ((uint32_t)(e + 7) << 3) | (uint32_t)(mant >> 49);
        const unsigned long long rem = mant & ((1ull << 49) - 1ull), half = 1ull << 48;
        if (rem > half || (rem == half && (q & 1u))) ++q;
        return (uint8_t)(sign | (q > 0x7Eu ? 0x7Eu : q));
    }
    return (uint8_t)(sign | (uint8_t)__double2int_rn(a * 512.0));  // exact scaling, then nearest even
}

// Value of an e4m3 code (the NaN codes are never written).
__device__ __forceinline__ double e4m3_to_f64(uint32_t c) {
    const int e = (int)((c >> 3) & 15u), m = (int)(c & 7u);
    const double v = e == 0 ? (double)m * 0x1p-9 : ldexp((double)(8 + m), e - 10);
    return (c & 0x80u) ? -v : v;
}

template <typename T>
__host__ __device__ __forceinline__ T ceil_div(T a, T b) { return (a + b - 1) / b; }

}  // namespace lsa

// Host-side launch helpers (defined in lsa_api.cu).
namespace lsa {
lsa_status set_error(lsa_status st, const char* fmt, ...);
lsa_status check_launch(const char* what);
int num_sms();

// Kernel timing: while lsa_timing_begin() is in effect, the launch inside a
// KTime's scope is bracketed by two CUDA events on its stream, filed under
// `name` (read back with lsa_timing_get).  Otherwise it does nothing.
struct KTime {
    int rec = -1, slot = -1;
    cudaStream_t st = nullptr;
    KTime(const char* name, cudaStream_t s);
    ~KTime();
};
}  // namespace lsa
