// softmax_math.cuh -- packed fp32 arithmetic of sm_100 for the softmax warps.
//
// Blackwell executes two fp32 FMAs or adds in one instruction (fma.rn.f32x2,
// add.rn.f32x2 on a 64-bit register pair) and takes the maximum of
// three operands in one instruction (max.f32 with three sources).  The softmax of a
// 128-column row spends most of its issue slots on exactly these operations, so using
// them halves the instruction count of the max, scale-and-shift and row-sum steps.
// Each packed operation rounds every lane exactly as the scalar instruction does.
#pragma once

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (a.x * b.x + c.x, a.y * b.y + c.y), each rounded to nearest even
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Maximum of x[0..N) (N a multiple of 16, at least 32): eight independent chains of
// three-input maxima, then a three-level reduction.
template <int N>
__device__ __forceinline__ float row_max(const float (&x)[N]) {
    static_assert(N % 16 == 0 && N >= 32, "row length");
    float m[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) m[t] = fmaxf(x[t], x[t + 8]);
#pragma unroll
    for (int c = 16; c < N; c += 16)
#pragma unroll
        for (int t = 0; t < 8; ++t) m[t] = max3f(m[t], x[c + 2 * t], x[c + 2 * t + 1]);
    return fmaxf(max3f(m[0], m[1], m[2]), max3f(max3f(m[3], m[4], m[5]), m[6], m[7]));
}

