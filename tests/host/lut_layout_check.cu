// Host-side check of the few-token table kernel's shared-memory layout rules
// (csrc/decode_lut.cuh), run by tests/test_lut_layout_cpu.py.  Prints "ok" or the
// first rule that fails.
#include <cstdio>
#include "decode_lut.cuh"

using namespace qlora;

static int fail(const char* what, int a, int b) {
  std::printf("FAIL %s (%d, %d)\n", what, a, b);
  return 1;
}

int main() {
  for (int k = 64; k <= 65536; k += 64) {
    const int rs = lut_row_stride(k);
    // a tile row: all K/2 code bytes, 16-byte multiple (bulk copy), 8 mod 32 words (a half
    // warp's 8-byte loads from 8 rows x 2 words fall in 16 distinct bank pairs)
    if (rs < k / 2 || rs % 16 != 0 || (rs / 4) % 32 != 8) return fail("row stride", k, rs);
    // an X row in halves: K values, 16-byte multiple, rows of different tokens in different banks
    const int xs = lut_x_stride(k);
    if (xs < k || (xs * 2) % 16 != 0 || ((xs * 2 / 4) % 32) == 0) return fail("x stride", k, xs);
  }
  for (int kb = 1; kb <= 1024; ++kb) {
    const int ss = lut_scale_stride(kb);
    // scale rows: every block, 16-byte aligned quads, 8 rows in 8 distinct groups of 4 banks
    if (ss < kb || ss % 4 != 0 || ss % 32 != 4) return fail("scale stride", kb, ss);
  }
  const int ms[] = {1, 2, 3, 4, 8};
  const int ks[] = {64, 1088, 4096, 11008};
  for (int m : ms)
    for (int k : ks)
      for (int t = 1; t <= 10; ++t)
        for (int slots = 1; slots <= kLutMaxSlots; ++slots)
          for (int single = 0; single <= 1; ++single) {
            const int r = 64;
            const LutLayout L = lut_layout(m, k, t, slots, r, single != 0);
            const int rows = t * kLutTile, kb = k / 64;
            const int off[] = {L.ring, L.consts, L.s2g, L.c1, L.x, L.xsc, L.part, L.u, L.b, L.bars, L.abort_word};
            for (int i = 0; i < 11; ++i)
              if (off[i] % 16 != 0) return fail("region alignment", i, off[i]);
            // each region holds what the kernel puts there, and regions do not overlap
            if (L.ring < kLutTableBytes) return fail("table", m, k);
            if (L.consts - L.ring < slots * kLutTile * lut_row_stride(k)) return fail("ring", m, k);
            if (L.s2g - L.consts < rows * kb * (single ? 4 : 1) + 16) return fail("consts", m, k);
            if (L.c1 - L.s2g < (single ? 0 : (rows * kb - 1) / 256 + 2) * 4) return fail("group scales", m, k);
            if (L.x - L.c1 < rows * lut_scale_stride(kb) * 4) return fail("c1", m, k);
            if (L.xsc - L.x < m * lut_x_stride(k) * 2) return fail("x", m, k);
            if (L.part - L.xsc < m * lut_scale_stride(kb) * 4) return fail("x scales", m, k);
            if (L.u - L.part < rows * m * kLutPartStride * 4) return fail("partials", m, k);
            if (L.b - L.u < m * r * 4) return fail("u", m, k);
            if (L.bars - L.b < rows * r * 2) return fail("b rows", m, k);
            if (L.abort_word - L.bars < (2 * kLutMaxSlots + 2) * 8) return fail("barriers", m, k);
            if (L.total - L.abort_word < 8) return fail("abort word", m, k);
          }
  std::printf("ok\n");
  return 0;
}
