// Fiber runtime of the test-only host emulation: one cluster at a time (cluster_size CTAs, default
// 1), each of its threads a ucontext.  Block, warp and cluster barriers block a fiber until every
// participant has arrived.  A deadlock, a write past a CTA's shared memory or a DSMEM address
// outside it aborts.  Host arrays from emu_alloc end against an inaccessible page, so reads or
// writes past their end fault.
#include <sys/mman.h>
#include <ucontext.h>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <vector>
#include "prelude.h"

namespace emu {
uint3 tid_, bid_;
dim3 bdim_, gdim_;
int cluster_size = 1;
namespace {
struct Fiber {
  ucontext_t ctx;
  bool done = false;
  int cta = 0;
  unsigned ltid = 0;
  std::vector<char> stack;
};
struct Barrier {
  long gen = 0;
  int arrived = 0;
  int acc = 0, result = 0;
};
std::vector<Fiber> fibers;
ucontext_t sched;
int cur = -1, per_cta = 0;
long progress = 0;
std::vector<Barrier> cta_bar, warp_bar;
Barrier cl_bar;
std::vector<uint64_t> xbuf;
std::vector<std::map<int, std::vector<float4>>> statics;  // per CTA: static shared declarations
std::function<void()>* body_ptr = nullptr;
std::vector<std::vector<float4>> bufs;
size_t smem_size = 0;
unsigned cluster_base = 0;

void yield_() { swapcontext(&fibers[cur].ctx, &sched); }
void trampoline() {
  (*body_ptr)();
  fibers[cur].done = true;
  ++progress;
  swapcontext(&fibers[cur].ctx, &sched);
}
int wait_on(Barrier& b, int n, int p) {
  b.acc |= (p != 0);
  const long g = b.gen;
  ++progress;
  if (++b.arrived == n) {
    b.arrived = 0;
    b.result = b.acc;
    b.acc = 0;
    ++b.gen;
    return b.result;
  }
  while (b.gen == g) yield_();
  return b.result;
}
}  // namespace

void syncthreads() { (void)wait_on(cta_bar[fibers[cur].cta], per_cta, 0); }
int syncthreads_or(int p) { return wait_on(cta_bar[fibers[cur].cta], per_cta, p); }
void syncwarp() { (void)wait_on(warp_bar[cur / 32], 32, 0); }
void cluster_sync() { (void)wait_on(cl_bar, (int)fibers.size(), 0); }
unsigned cluster_rank() { return (unsigned)fibers[cur].cta; }
void* cluster_map(void* p, unsigned rank) {
  const char* own = reinterpret_cast<const char*>(bufs[fibers[cur].cta].data());
  const ptrdiff_t off = reinterpret_cast<const char*>(p) - own;
  if (off < 0 || (size_t)off >= smem_size || rank >= (unsigned)cluster_size) {
    fprintf(stderr, "emu: DSMEM map of offset %td (smem %zu) to rank %u of %d\n", off, smem_size, rank, cluster_size);
    abort();
  }
  return reinterpret_cast<char*>(bufs[rank].data()) + off;
}
uint64_t xchg(uint64_t bits, int src, bool xor_mode) {
  const int me = cur;
  const int lane = me & 31;
  xbuf[me] = bits;
  (void)wait_on(warp_bar[me / 32], 32, 0);
  const int from = (me & ~31) | ((xor_mode ? (lane ^ src) : src) & 31);
  const uint64_t r = xbuf[from];
  (void)wait_on(warp_bar[me / 32], 32, 0);
  return r;
}
float4* smem() { return bufs[fibers[cur].cta].data(); }
void* shared_static_bytes(int id, size_t bytes) {
  std::vector<float4>& v = statics[fibers[cur].cta][id];
  const size_t n = (bytes + sizeof(float4) - 1) / sizeof(float4);
  if (v.size() != n) {
    v.assign(n, float4());
    memset(v.data(), 0xFF, n * sizeof(float4));  // NaN: unwritten reads show up
  }
  return v.data();
}
unsigned ballot(int p) {
  const int me = cur;
  xbuf[me] = p ? 1 : 0;
  (void)wait_on(warp_bar[me / 32], 32, 0);
  unsigned mask = 0;
  for (int l = 0; l < 32; ++l)
    if (xbuf[(me & ~31) | l]) mask |= 1u << l;
  (void)wait_on(warp_bar[me / 32], 32, 0);
  return mask;
}
int lane_id() { return cur & 31; }
unsigned match_any(unsigned long long v) {
  const int me = cur;
  xbuf[me] = v;
  (void)wait_on(warp_bar[me / 32], 32, 0);
  unsigned mask = 0;
  for (int l = 0; l < 32; ++l)
    if (xbuf[(me & ~31) | l] == v) mask |= 1u << l;
  (void)wait_on(warp_bar[me / 32], 32, 0);
  return mask;
}

void launch(dim3 grid, dim3 block, size_t smem_bytes, std::function<void()> body) {
  per_cta = (int)(block.x * block.y * block.z);
  if (per_cta % 32) {
    fprintf(stderr, "emu: block size %d is not a multiple of 32\n", per_cta);
    abort();
  }
  const int cs = cluster_size;
  if (grid.x % cs) {
    fprintf(stderr, "emu: grid.x %u is not a multiple of the cluster size %d\n", grid.x, cs);
    abort();
  }
  bdim_ = block;
  gdim_ = grid;
  smem_size = smem_bytes;
  const size_t guard = 4096;
  bufs.assign(cs, std::vector<float4>((smem_bytes + guard) / sizeof(float4) + 1));
  const int n = cs * per_cta;
  for (unsigned bz = 0; bz < grid.z; ++bz)
    for (unsigned by = 0; by < grid.y; ++by)
      for (unsigned bx0 = 0; bx0 < grid.x; bx0 += cs) {
        cluster_base = bx0;
        for (int c = 0; c < cs; ++c) {
          unsigned char* raw = reinterpret_cast<unsigned char*>(bufs[c].data());
          memset(raw, 0xFF, smem_bytes);          // NaN: unstaged reads show up
          memset(raw + smem_bytes, 0xAB, guard);  // canary past the requested size
        }
        fibers.clear();
        fibers.resize(n);
        cta_bar.assign(cs, Barrier());
        warp_bar.assign(n / 32, Barrier());
        cl_bar = Barrier();
        xbuf.assign(n, 0);
        statics.assign(cs, {});
        body_ptr = &body;
        for (int i = 0; i < n; ++i) {
          Fiber& f = fibers[i];
          f.cta = i / per_cta;
          f.ltid = (unsigned)(i % per_cta);
          f.stack.resize(1 << 16);
          getcontext(&f.ctx);
          f.ctx.uc_stack.ss_sp = f.stack.data();
          f.ctx.uc_stack.ss_size = f.stack.size();
          f.ctx.uc_link = &sched;
          makecontext(&f.ctx, trampoline, 0);
        }
        for (;;) {
          bool any = false;
          const long before = progress;
          for (int i = 0; i < n; ++i) {
            if (fibers[i].done) continue;
            any = true;
            cur = i;
            const unsigned lt = fibers[i].ltid;
            tid_ = make_uint3(lt % block.x, (lt / block.x) % block.y, lt / (block.x * block.y));
            bid_ = make_uint3(bx0 + fibers[i].cta, by, bz);
            swapcontext(&sched, &fibers[i].ctx);
          }
          if (!any) break;
          if (progress == before) {
            fprintf(stderr, "emu: deadlock in cluster at block (%u,%u,%u)\n", bx0, by, bz);
            abort();
          }
        }
        for (int c = 0; c < cs; ++c) {
          const unsigned char* raw = reinterpret_cast<const unsigned char*>(bufs[c].data());
          for (size_t i = 0; i < guard; ++i)
            if (raw[smem_bytes + i] != 0xAB) {
              fprintf(stderr, "emu: shared-memory overflow past %zu bytes in block %u\n", smem_bytes, bx0 + c);
              abort();
            }
        }
      }
}
}  // namespace emu

// Arrays that end flush against a PROT_NONE page, so reads or writes past the end fault.
static std::map<void*, std::pair<void*, size_t>> g_maps;
extern "C" void* emu_alloc(size_t bytes) {
  const size_t page = 4096, sz = (bytes + 15) & ~size_t(15), data_pages = (sz + page - 1) / page;
  const size_t total = (data_pages + 2) * page;
  char* base = static_cast<char*>(mmap(nullptr, total, PROT_READ | PROT_WRITE, MAP_PRIVATE | MAP_ANONYMOUS, -1, 0));
  if (base == MAP_FAILED) return nullptr;
  mprotect(base, page, PROT_NONE);
  mprotect(base + (data_pages + 1) * page, page, PROT_NONE);
  char* p = base + (data_pages + 1) * page - sz;
  memset(p, 0xFF, sz);
  g_maps[p] = {base, total};
  return p;
}
extern "C" void emu_free(void* p) {
  auto it = g_maps.find(p);
  if (it != g_maps.end()) {
    munmap(it->second.first, it->second.second);
    g_maps.erase(it);
  }
}
