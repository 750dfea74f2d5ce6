// Workspace of a decode call: the sequence records that the decode grid writes for the
// combine grid, and the split partials (see the Schedule comment in mla_internal.h; the
// decode CTAs derive their page ranges themselves, worker_range.cuh).
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {

size_t carve_schedule(void* base, int batch, int heads, int num_workers, Schedule* s) {
  auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 0;
  char* p = static_cast<char*>(base);
  auto take = [&](size_t bytes) {
    void* r = p ? p + off : nullptr;
    off = align(off + bytes);
    return r;
  };
  Schedule t;
  t.num_workers = num_workers;
  t.seq = static_cast<SeqInfo*>(take(sizeof(SeqInfo) * batch));
  t.part_lse = static_cast<float*>(take(sizeof(float) * 2 * (size_t)num_workers * heads));
  t.part_o = static_cast<float*>(take(sizeof(float) * 2 * (size_t)num_workers * heads * kDLatent));
  if (s) *s = t;
  return off;
}

}  // namespace mla
