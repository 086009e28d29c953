// Pieces shared by the tensor-core latent decode kernels (MLA, GLA, MLRA).
#pragma once

#include "kvattn_internal.cuh"
#include "sm100.cuh"

namespace kvattn {
namespace latent {

constexpr int kRows = 128;                 // MMA M: query-head rows
constexpr int kQChunkBytes = kRows * 128;  // 128 rows x 64 bf16, 128-byte swizzle
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kRescaleThreshold = 8.f;   // log2 units: O is rescaled only past 2^8
constexpr int kMaxSplitPages = 1024;       // pages per part the page-validity table holds

// 2^x on the special-function unit (ex2.approx.ftz: ~2 ulp, subnormal results
// flushed to zero, 2^-inf = 0); the softmax weights are rounded to bf16 next
__device__ __forceinline__ float exp2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// d = a * b + c on two fp32 lanes at once (one packed FMA instruction)
__device__ __forceinline__ void ffma2(float &dx, float &dy, float ax, float ay, float bx, float by, float cx, float cy)
{
    asm("{\n\t.reg .b64 a2, b2, c2, d2;\n\tmov.b64 a2, {%2, %3};\n\tmov.b64 b2, {%4, %5};\n\tmov.b64 c2, {%6, %7};\n\t"
        "fma.rn.f32x2 d2, a2, b2, c2;\n\tmov.b64 {%0, %1}, d2;\n\t}"
        : "=f"(dx), "=f"(dy)
        : "f"(ax), "f"(ay), "f"(bx), "f"(by), "f"(cx), "f"(cy));
}

// d = a + b on two fp32 lanes at once
__device__ __forceinline__ void fadd2(float &dx, float &dy, float ax, float ay, float bx, float by)
{
    asm("{\n\t.reg .b64 a2, b2, d2;\n\tmov.b64 a2, {%2, %3};\n\tmov.b64 b2, {%4, %5};\n\t"
        "add.rn.f32x2 d2, a2, b2;\n\tmov.b64 {%0, %1}, d2;\n\t}"
        : "=f"(dx), "=f"(dy)
        : "f"(ax), "f"(ay), "f"(bx), "f"(by));
}

// three-input maximum and minimum
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float fmin3(float a, float b, float c)
{
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Maximum (kMax) or minimum of n values, n a multiple of 8.
template <bool kMax, int n>
__device__ __forceinline__ float reduce_extreme(const float *v)
{
    static_assert(n % 8 == 0, "multiple of 8");
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        acc[q] = v[q];
#pragma unroll
        for (int i = q + 8; i < n; i += 16) {
            if (i + 8 < n)
                acc[q] = kMax ? fmax3(acc[q], v[i], v[i + 8]) : fmin3(acc[q], v[i], v[i + 8]);
            else
                acc[q] = kMax ? fmaxf(acc[q], v[i]) : fminf(acc[q], v[i]);
        }
    }
    const float x = kMax ? fmax3(acc[0], acc[1], acc[2]) : fmin3(acc[0], acc[1], acc[2]);
    const float y = kMax ? fmax3(acc[3], acc[4], acc[5]) : fmin3(acc[3], acc[4], acc[5]);
    const float z = kMax ? fmaxf(acc[6], acc[7]) : fminf(acc[6], acc[7]);
    return kMax ? fmax3(x, y, z) : fmin3(x, y, z);
}

__device__ __forceinline__ long long page_id(const DecodeArgs &a, int b, int pi) { return row_page(a, b, pi); }

__device__ __forceinline__ bool page_ok(const DecodeArgs &a, long long page)
{
    return page >= 0 && page < a.num_pages;
}

// Context tokens in tile j of the part starting at page p0 (0 if one of its
// pages has a bad id); pvalid holds one bit per page of the part.
template <int T>
__device__ __forceinline__ int tile_ntok(const uint32_t *pvalid, int L, int p0, int j)
{
    constexpr int kSubs = T >= kPage ? T / kPage : 1;     // pages a tile spans
    const int tok0 = p0 * kPage + j * T;
    const int ntok = min(T, L - tok0);
    bool ok = true;
#pragma unroll
    for (int sub = 0; sub < kSubs; ++sub) {
        const int pg = (j * T) / kPage + sub;
        if (sub * kPage < ntok)
            ok = ok && ((pvalid[pg >> 5] >> (pg & 31)) & 1u);
    }
    return ok ? ntok : 0;
}

// Fill the page-validity bits of a part (threads [first, first + count)).
__device__ __forceinline__ void fill_page_bits(uint32_t *pvalid, const DecodeArgs &a, int b, int p0, int npg,
                                               int tid, int count)
{
    for (int w = tid; w < (npg + 31) / 32; w += count) {
        uint32_t bits = 0;
        for (int i = 32 * w; i < min(npg, 32 * w + 32); ++i)
            bits |= (page_ok(a, page_id(a, b, p0 + i)) ? 1u : 0u) << (i & 31);
        pvalid[w] = bits;
    }
}

}  // namespace latent
}  // namespace kvattn
