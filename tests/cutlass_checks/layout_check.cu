// Host-only check of the tcgen05 attention kernel's shared-memory tiles: are
// they canonical UMMA layouts?  CuTe's 128-byte-swizzle atoms, tiled in the
// kernel's order, must place every element at the byte offset the kernel's
// writers (TMA boxes, swz()) use.  CuTe's composed layouts apply the swizzle
// to the shared-memory byte address, so the inner layout is evaluated and the
// swizzle (bits 4-6 ^= bits 7-9) applied to the byte offset.
#include <cstdio>
#include <cute/tensor.hpp>
#include <cute/atom/mma_traits_sm100.hpp>
using namespace cute;

static int ours(int half_bytes, int row, int col) {   // [col / 64][rows x 128 B], swizzled
  return (col / 64) * half_bytes + row * 128 + ((((col % 64) / 8) ^ (row & 7)) << 4) + 2 * (col % 8);
}

int main() {
  using T = cute::bfloat16_t;
  int bad = 0;
  // K-major operands (Q: 128 columns x 128 dims, halves 16 KiB apart; K: 64 tokens x 128 dims, halves 8 KiB;
  // P: 128 columns x 64 tokens).  One 64-element-wide half: rows in 8-row atoms, atoms stacked along M.
  {
    auto lay = tile_to_shape(UMMA::Layout_K_SW128_Atom<T>{}, Shape<_128, _64>{});
    for (int m = 0; m < 128; ++m)
      for (int k = 0; k < 64; ++k) {
        int a = int(lay.layout_b()(m, k)) * 2; int cute_bytes = a ^ (((a >> 7) & 7) << 4);
        if (cute_bytes != ours(0, m, k)) { if (bad++ < 5) printf("K-major m=%d k=%d cute=%d ours=%d\n", m, k, cute_bytes, ours(0, m, k)); }
      }
    printf("K-major (128 x 64): %s\n", bad ? "MISMATCH" : "equal");
  }
  // MN-major V: element (dim n, token t) of a 64-token tile; dims 0-63 and 64-127 in halves 8 KiB
  // apart, tokens in 8-row atoms stacked along K first.  Tile the atom K-first, then MN.
  {
    int bad2 = 0;
    auto atom = UMMA::Layout_MN_SW128_Atom<T>{};
    auto lay = tile_to_shape(atom, Shape<_128, _64>{}, Step<_2, _1>{});
    for (int n = 0; n < 128; ++n)
      for (int t = 0; t < 64; ++t) {
        int a = int(lay.layout_b()(n, t)) * 2; int cute_bytes = a ^ (((a >> 7) & 7) << 4);
        int o = ours(64 * 128, t, n);
        if (cute_bytes != o) { if (bad2++ < 5) printf("MN-major n=%d t=%d cute=%d ours=%d\n", n, t, cute_bytes, o); }
      }
    printf("MN-major (128 x 64, K first): %s\n", bad2 ? "MISMATCH" : "equal");
    bad += bad2;
  }
  return bad ? 1 : 0;
}
