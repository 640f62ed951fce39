// streamer.cpp -- pinned-host NF4 base -> 2-slot VRAM ring, prefetched one
// block ahead on a dedicated copy stream.
//
// HN comment (host-RAM base, prefetch-one-ahead ring): the frozen base sits
// in host RAM and streams into a small pool of pre-allocated VRAM buffers
// one decoder layer at a time, prefetched one ahead on a dedicated CUDA
// stream.  Poros API reference: block_size layers per block (default 4),
// enable_prefetch, and a block manager that keeps buffers alive across
// streams (there: record_stream; here: explicit CUDA events).
//
// Lifetime fences:
//   ready[slot]  recorded on the copy stream after a block's H2D copy; the
//                compute stream waits on it in acquire();
//   free[slot]   recorded on the compute stream in release(); the copy stream
//                waits on it before overwriting that slot.
// A slot's content is therefore never overwritten while kernels that read
// it are queued or running, and never read before its copy has landed,
// whatever the host timing.
#include <cuda_runtime.h>
#include <string.h>

#include <chrono>
#include <mutex>
#include <thread>
#include <vector>

#include "internal.h"

using namespace hsnf4;

namespace {

constexpr size_t kAlign = 1024;

size_t proj_codes_bytes(const hsnf4_layer_desc& d, int p) {
  return static_cast<size_t>(d.n_out[p]) * static_cast<size_t>(d.k_in[p]) / 2;
}
size_t proj_absmax_bytes(const hsnf4_layer_desc& d, int p) {
  return static_cast<size_t>(d.n_out[p]) * static_cast<size_t>(d.k_in[p]) / 64 * 4;
}
// slab bytes of projection p: NF4 codes then absmax, or the dense bf16
// weight, each range starting on a 1 KiB boundary
size_t proj_bytes(const hsnf4_layer_desc& d, int p) {
  if (d.base_format == HSNF4_BASE_BF16)
    return round_up(static_cast<size_t>(d.n_out[p]) * static_cast<size_t>(d.k_in[p]) * 2, kAlign);
  return round_up(proj_codes_bytes(d, p), kAlign) + round_up(proj_absmax_bytes(d, p), kAlign);
}

int check_layer(const char* fn, const hsnf4_layer_desc* d) {
  if (!d) return fail(HSNF4_ERR_INVALID, "%s: layer descriptor is NULL", fn);
  if (d->n_proj < 1 || d->n_proj > HSNF4_MAX_PROJ)
    return fail(HSNF4_ERR_INVALID, "%s: n_proj must be in [1, %d] (got %d)", fn, HSNF4_MAX_PROJ,
                d->n_proj);
  if (d->base_format != HSNF4_BASE_NF4 && d->base_format != HSNF4_BASE_BF16)
    return fail(HSNF4_ERR_INVALID, "%s: base_format must be HSNF4_BASE_NF4 or HSNF4_BASE_BF16 "
                "(got %d)", fn, d->base_format);
  for (int p = 0; p < d->n_proj; ++p)
    if (d->n_out[p] < 1 || d->k_in[p] < 64 || d->k_in[p] % 64)
      return fail(HSNF4_ERR_INVALID, "%s: projection %d has invalid shape %lld x %lld", fn, p,
                  (long long)d->n_out[p], (long long)d->k_in[p]);
  return HSNF4_OK;
}

size_t layer_bytes(const hsnf4_layer_desc& d) {
  size_t b = 0;
  for (int p = 0; p < d.n_proj; ++p) b += proj_bytes(d, p);
  return b;
}

void layer_offsets(const hsnf4_layer_desc& d, int proj, size_t* co, size_t* ao) {
  size_t off = 0;
  for (int p = 0; p < proj; ++p) off += proj_bytes(d, p);
  *co = off;
  *ao = (d.base_format == HSNF4_BASE_BF16) ? off : off + round_up(proj_codes_bytes(d, proj), kAlign);
}

enum SlotState { kEmpty = 0, kLoaded = 1, kAcquired = 2, kReleased = 3 };

struct Slot {
  int block = -1;
  SlotState state = kEmpty;
  bool free_recorded = false;
  uint64_t last_use = 0;
  cudaEvent_t ready = nullptr, free = nullptr;
};

}  // namespace

struct hsnf4_streamer {
  const uint8_t* slab = nullptr;
  size_t slab_bytes = 0;
  std::vector<hsnf4_layer_desc> layers;
  std::vector<size_t> layer_off, layer_size;
  std::vector<size_t> shard_off;  // shard_slab: where block b's shard sits in the slab
  hsnf4_stream_config cfg{};
  uint8_t* ring = nullptr;
  size_t slot_bytes = 0;
  cudaStream_t copy = nullptr;
  int n_blocks = 0;
  std::vector<Slot> slots;
  uint64_t seq = 0;
  hsnf4_stream_stats stats{};
  std::mutex mu;

  int first_layer(int b) const { return b * cfg.block_size; }
  int end_layer(int b) const {
    const int e = (b + 1) * cfg.block_size;
    return e < static_cast<int>(layers.size()) ? e : static_cast<int>(layers.size());
  }
  size_t block_off(int b) const { return layer_off[first_layer(b)]; }
  size_t block_bytes(int b) const {
    const int l = end_layer(b) - 1;
    return layer_off[l] + layer_size[l] - layer_off[first_layer(b)];
  }
  // Slot holding block b in `state`, or -1.
  int find(int b, SlotState state) const {
    for (int i = 0; i < static_cast<int>(slots.size()); ++i)
      if (slots[i].block == b && slots[i].state == state) return i;
    return -1;
  }
};

namespace {

int record(cudaEvent_t ev, cudaStream_t st, const char* what) {
  if (take_fault(kFaultEventRecord))
    return fail(HSNF4_ERR_CUDA, "%s: injected fault at event_record", what);
  return cuda_status(cudaEventRecord(ev, st), what);
}

// Enqueue the copy of block b into slot i (caller holds the lock).
// `after` (may be null): a stream whose queued work the copy must follow.
int enqueue_copy(hsnf4_streamer* s, int i, int b, cudaStream_t after) {
  Slot& sl = s->slots[i];
  int rc;
  if (sl.free_recorded) {
    rc = cuda_status(cudaStreamWaitEvent(s->copy, sl.free, 0), "prefetch: wait slot free");
    if (rc) return rc;
  }
  if (after) {
    // no-prefetch mode: the copy also waits for all compute queued so far
    rc = record(sl.ready, after, "acquire: order copy after compute");
    if (rc) return rc;
    rc = cuda_status(cudaStreamWaitEvent(s->copy, sl.ready, 0), "acquire: wait compute");
    if (rc) return rc;
  }
  if (take_fault(kFaultCopyEnqueue))
    return fail(HSNF4_ERR_CUDA, "prefetch: injected fault at copy_enqueue (block %d)", b);
  const size_t bytes = s->block_bytes(b);
  uint8_t* slot = s->ring + static_cast<size_t>(i) * s->slot_bytes;
  size_t copied = bytes;
  if (s->cfg.gather) {
    // sharded: this rank's shard over its own link, then the gather fills
    // the other ranks' shards, in copy-stream order before `ready`
    const int world = s->cfg.shard_world > 1 ? s->cfg.shard_world : 1;
    size_t S = 0, off = 0, len = 0;
    stream_shard_range(bytes, world, s->cfg.shard_rank, &S, &off, &len);
    if (len) {
      // the whole stack in the slab, or (shard_slab) only this rank's shards
      const uint8_t* src =
          s->cfg.shard_slab ? s->slab + s->shard_off[b] : s->slab + s->block_off(b) + off;
      rc = cuda_status(cudaMemcpyAsync(slot + off, src, len, cudaMemcpyHostToDevice, s->copy),
                       "prefetch: cudaMemcpyAsync H2D (shard)");
      if (rc) return rc;
    }
    const int g = s->cfg.gather(slot, S, world, b, s->copy, s->cfg.gather_user);
    if (g != 0)
      return fail(HSNF4_ERR_CUDA, "prefetch: gather of block %d failed (callback returned %d)",
                  b, g);
    s->stats.gathers += 1;
    copied = len;
  } else {
    rc = cuda_status(cudaMemcpyAsync(slot, s->slab + s->block_off(b), bytes,
                                     cudaMemcpyHostToDevice, s->copy),
                     "prefetch: cudaMemcpyAsync H2D");
    if (rc) return rc;
  }
  rc = record(sl.ready, s->copy, "prefetch: record ready");
  if (rc) return rc;
  sl.block = b;
  sl.state = kLoaded;
  s->stats.h2d_bytes += copied;
  s->stats.copies += 1;
  return HSNF4_OK;
}

// Pick the slot a new copy of block b goes to: an empty slot, else a
// released slot -- the one whose block is needed furthest in the future
// according to `upcoming` (blocks not listed count as never needed; ties go
// to the least recently used).  Returns -1 (detail set unless quiet) if
// every slot holds a block that is prefetched or in use.
int choose_slot(hsnf4_streamer* s, int b, const int* upcoming = nullptr, int n_up = 0,
                bool quiet = false) {
  int best = -1, best_next = -1;
  for (int i = 0; i < static_cast<int>(s->slots.size()); ++i) {
    const Slot& sl = s->slots[i];
    if (sl.state == kEmpty) return i;
    if (sl.state != kReleased) continue;
    int next = 1 << 30;  // not needed within the window
    for (int k = 0; k < n_up; ++k)
      if (upcoming[k] == sl.block) {
        next = k;
        break;
      }
    if (best < 0 || next > best_next ||
        (next == best_next && sl.last_use < s->slots[best].last_use)) {
      best = i;
      best_next = next;
    }
  }
  if (best < 0 && !quiet)
    fail(HSNF4_ERR_STATE,
         "prefetch(%d): no free slot -- all %zu slots hold blocks that are prefetched or "
         "acquired and not released; release before prefetching further ahead",
         b, s->slots.size());
  return best;
}

int check_block(const char* fn, const hsnf4_streamer* s, int b) {
  if (!s) return fail(HSNF4_ERR_INVALID, "%s: streamer is NULL", fn);
  if (b < 0 || b >= s->n_blocks)
    return fail(HSNF4_ERR_INVALID, "%s: block %d out of range [0, %d)", fn, b, s->n_blocks);
  return HSNF4_OK;
}

}  // namespace

extern "C" {

int stream_layer_bytes(const hsnf4_layer_desc* layer, size_t* out_bytes) {
  int rc = check_layer("stream_layer_bytes", layer);
  if (rc) return rc;
  if (!out_bytes) return fail(HSNF4_ERR_INVALID, "stream_layer_bytes: out_bytes is NULL");
  *out_bytes = layer_bytes(*layer);
  return HSNF4_OK;
}

int stream_layer_offsets(const hsnf4_layer_desc* layer, int proj, size_t* codes_off,
                         size_t* absmax_off) {
  int rc = check_layer("stream_layer_offsets", layer);
  if (rc) return rc;
  if (proj < 0 || proj >= layer->n_proj)
    return fail(HSNF4_ERR_INVALID, "stream_layer_offsets: proj %d out of range", proj);
  if (!codes_off || !absmax_off)
    return fail(HSNF4_ERR_INVALID, "stream_layer_offsets: output pointer is NULL");
  layer_offsets(*layer, proj, codes_off, absmax_off);
  return HSNF4_OK;
}

int stream_slab_bytes(const hsnf4_layer_desc* layers, int n_layers, size_t* out_bytes) {
  if (!layers || n_layers < 1 || !out_bytes)
    return fail(HSNF4_ERR_INVALID, "stream_slab_bytes: need layers, n_layers >= 1, out_bytes");
  size_t total = 0;
  for (int l = 0; l < n_layers; ++l) {
    int rc = check_layer("stream_slab_bytes", &layers[l]);
    if (rc) return rc;
    total += layer_bytes(layers[l]);
  }
  *out_bytes = total;
  return HSNF4_OK;
}

int stream_slot_bytes(const hsnf4_layer_desc* layers, int n_layers, int block_size,
                      size_t* out_bytes) {
  size_t ring = 0;
  int rc = stream_ring_bytes(layers, n_layers, block_size, &ring);
  if (rc) return rc;
  *out_bytes = ring / 2;
  return HSNF4_OK;
}

int stream_shard_range(size_t block_bytes, int world, int rank, size_t* shard_bytes,
                       size_t* off, size_t* len) {
  if (world < 1 || rank < 0 || rank >= world || !shard_bytes || !off || !len)
    return fail(HSNF4_ERR_INVALID, "stream_shard_range: need 0 <= rank < world and outputs "
                "(world=%d rank=%d)", world, rank);
  const size_t S = round_up((block_bytes + world - 1) / world, kAlign);
  const size_t o = S * static_cast<size_t>(rank);
  *shard_bytes = S;
  *off = o;
  *len = o >= block_bytes ? 0 : (block_bytes - o < S ? block_bytes - o : S);
  return HSNF4_OK;
}

int stream_slot_bytes_sharded(const hsnf4_layer_desc* layers, int n_layers, int block_size,
                              int world, size_t* out_bytes) {
  if (!layers || n_layers < 1 || !out_bytes || block_size < 1 || world < 1)
    return fail(HSNF4_ERR_INVALID, "stream_slot_bytes_sharded: need layers, n_layers >= 1, "
                "block_size >= 1, world >= 1, out_bytes");
  size_t slot = 0;
  for (int first = 0; first < n_layers; first += block_size) {
    size_t b = 0;
    for (int l = first; l < n_layers && l < first + block_size; ++l) {
      int rc = check_layer("stream_slot_bytes_sharded", &layers[l]);
      if (rc) return rc;
      b += layer_bytes(layers[l]);
    }
    size_t S = 0, off = 0, len = 0;
    stream_shard_range(b, world, 0, &S, &off, &len);
    if (S * world > slot) slot = S * world;
  }
  *out_bytes = slot;
  return HSNF4_OK;
}

int stream_shard_slab_layout(const hsnf4_layer_desc* layers, int n_layers, int block_size,
                             int world, int rank, int block, size_t* block_off, size_t* len,
                             size_t* total_bytes) {
  static const char* fn = "stream_shard_slab_layout";
  if (!layers || n_layers < 1 || block_size < 1 || world < 1 || rank < 0 || rank >= world)
    return fail(HSNF4_ERR_INVALID, "%s: need layers, n_layers >= 1, block_size >= 1 and "
                "0 <= rank < world (got rank %d of %d)", fn, rank, world);
  const int n_blocks = (n_layers + block_size - 1) / block_size;
  if (block < -1 || block >= n_blocks)
    return fail(HSNF4_ERR_INVALID, "%s: block %d outside [-1, %d)", fn, block, n_blocks);
  size_t at = 0, found_off = 0, found_len = 0;
  for (int b = 0; b < n_blocks; ++b) {
    size_t bytes = 0;
    for (int l = b * block_size; l < n_layers && l < (b + 1) * block_size; ++l) {
      int rc = check_layer(fn, &layers[l]);
      if (rc) return rc;
      bytes += layer_bytes(layers[l]);
    }
    size_t S = 0, off = 0, n = 0;
    stream_shard_range(bytes, world, rank, &S, &off, &n);
    if (b == block) {
      found_off = at;
      found_len = n;
    }
    at += n;
  }
  if (block_off) *block_off = found_off;
  if (len) *len = found_len;
  if (total_bytes) *total_bytes = at;
  return HSNF4_OK;
}

int stream_ring_bytes(const hsnf4_layer_desc* layers, int n_layers, int block_size,
                      size_t* out_bytes) {
  if (!layers || n_layers < 1 || !out_bytes || block_size < 1)
    return fail(HSNF4_ERR_INVALID,
                "stream_ring_bytes: need layers, n_layers >= 1, block_size >= 1, out_bytes");
  size_t slot = 0;
  for (int first = 0; first < n_layers; first += block_size) {
    size_t b = 0;
    for (int l = first; l < n_layers && l < first + block_size; ++l) {
      int rc = check_layer("stream_ring_bytes", &layers[l]);
      if (rc) return rc;
      b += layer_bytes(layers[l]);
    }
    if (b > slot) slot = b;
  }
  *out_bytes = 2 * slot;
  return HSNF4_OK;
}

int stream_create(const void* pinned_slab, size_t slab_bytes, const hsnf4_layer_desc* layers,
                  int n_layers, const hsnf4_stream_config* cfg, void* ring_dev, size_t ring_bytes,
                  void* copy_stream, hsnf4_streamer** out) {
  static const char* fn = "stream_create";
  if (!out || !pinned_slab || !layers || !cfg || !ring_dev || n_layers < 1)
    return fail(HSNF4_ERR_INVALID, "%s: NULL argument or n_layers < 1", fn);
  *out = nullptr;
  if (cfg->block_size < 1)
    return fail(HSNF4_ERR_INVALID, "%s: block_size must be >= 1 (got %d)", fn, cfg->block_size);
  if (reinterpret_cast<uintptr_t>(ring_dev) % kAlign)
    return fail(HSNF4_ERR_INVALID, "%s: ring must be %zu-byte aligned", fn, kAlign);
  const int n_slots = cfg->n_slots == 0 ? 2 : cfg->n_slots;
  if (n_slots < 2 || n_slots > HSNF4_MAX_SLOTS)
    return fail(HSNF4_ERR_INVALID, "%s: n_slots must be 0 (= 2) or in [2, %d] (got %d)", fn,
                HSNF4_MAX_SLOTS, cfg->n_slots);
  const int world = cfg->shard_world > 1 ? cfg->shard_world : 1;
  if (cfg->shard_world < 0 || cfg->shard_rank < 0 || cfg->shard_rank >= world)
    return fail(HSNF4_ERR_INVALID, "%s: need 0 <= shard_rank < shard_world (got rank %d of %d)",
                fn, cfg->shard_rank, cfg->shard_world);
  if (world > 1 && !cfg->gather)
    return fail(HSNF4_ERR_INVALID, "%s: a stream sharded over %d ranks needs a gather callback",
                fn, world);
  if (cfg->shard_slab && !cfg->gather)
    return fail(HSNF4_ERR_INVALID, "%s: shard_slab needs a sharded stream (a gather callback)",
                fn);
  size_t need_slab = 0, need_ring = 0;
  int rc = cfg->shard_slab
               ? stream_shard_slab_layout(layers, n_layers, cfg->block_size, world,
                                          cfg->shard_rank, -1, nullptr, nullptr, &need_slab)
               : stream_slab_bytes(layers, n_layers, &need_slab);
  if (rc) return rc;
  rc = cfg->gather
           ? stream_slot_bytes_sharded(layers, n_layers, cfg->block_size, world, &need_ring)
           : stream_slot_bytes(layers, n_layers, cfg->block_size, &need_ring);
  if (rc) return rc;
  const size_t slot_bytes = need_ring;
  need_ring *= static_cast<size_t>(n_slots);
  if (slab_bytes < need_slab)
    return fail(HSNF4_ERR_OOM, "%s: pinned slab too small: need %zu bytes, given %zu", fn,
                need_slab, slab_bytes);
  if (ring_bytes < need_ring)
    return fail(HSNF4_ERR_OOM,
                "%s: ring too small for block_size=%d and %d slots: need %zu bytes, given %zu "
                "(lower block_size to shrink the ring)",
                fn, cfg->block_size, n_slots, need_ring, ring_bytes);
  auto* s = new (std::nothrow) hsnf4_streamer();
  if (!s) return fail(HSNF4_ERR_OOM, "%s: host allocation failed", fn);
  s->slab = static_cast<const uint8_t*>(pinned_slab);
  s->slab_bytes = slab_bytes;
  s->layers.assign(layers, layers + n_layers);
  size_t off = 0;
  for (int l = 0; l < n_layers; ++l) {
    s->layer_off.push_back(off);
    s->layer_size.push_back(layer_bytes(layers[l]));
    off += s->layer_size.back();
  }
  s->cfg = *cfg;
  if (s->cfg.poison_on_release) s->cfg.reuse_resident = 0;  // poisoned data is never reused
  if (cfg->shard_slab) {
    const int nb = (n_layers + cfg->block_size - 1) / cfg->block_size;
    for (int b = 0; b < nb; ++b) {
      size_t o = 0;
      stream_shard_slab_layout(layers, n_layers, cfg->block_size, world, cfg->shard_rank, b, &o,
                               nullptr, nullptr);
      s->shard_off.push_back(o);
    }
  }
  s->ring = static_cast<uint8_t*>(ring_dev);
  s->slot_bytes = slot_bytes;
  s->slots.resize(static_cast<size_t>(n_slots));
  s->copy = static_cast<cudaStream_t>(copy_stream);
  s->n_blocks = (n_layers + cfg->block_size - 1) / cfg->block_size;
  for (auto& sl : s->slots) {
    rc = cuda_status(cudaEventCreateWithFlags(&sl.ready, cudaEventDisableTiming), "event create");
    if (!rc)
      rc = cuda_status(cudaEventCreateWithFlags(&sl.free, cudaEventDisableTiming), "event create");
    if (rc) {
      stream_destroy(s);
      return rc;
    }
  }
  *out = s;
  return HSNF4_OK;
}

int stream_num_blocks(const hsnf4_streamer* s) { return s ? s->n_blocks : 0; }

int stream_block_prefetch(hsnf4_streamer* s, int block) {
  int rc = check_block("stream_block_prefetch", s, block);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(s->mu);
  // Already copied and not yet consumed: nothing to do.
  if (s->find(block, kLoaded) >= 0) {
    s->stats.reuses += 1;
    return HSNF4_OK;
  }
  // Still resident from an earlier acquire (the forward/backward turn-around).
  if (s->cfg.reuse_resident) {
    const int rel = s->find(block, kReleased);
    if (rel >= 0) {
      s->slots[rel].state = kLoaded;
      s->stats.reuses += 1;
      return HSNF4_OK;
    }
    if (s->find(block, kAcquired) >= 0) {
      s->stats.reuses += 1;
      return HSNF4_OK;
    }
  }
  if (!s->cfg.enable_prefetch) return HSNF4_OK;  // acquire() issues the copy
  const int i = choose_slot(s, block);
  if (i < 0) return HSNF4_ERR_STATE;
  return enqueue_copy(s, i, block, nullptr);
}

int stream_prefetch_ahead(hsnf4_streamer* s, const int* upcoming, int n, int* issued) {
  if (issued) *issued = 0;
  if (!s || (!upcoming && n > 0) || n < 0)
    return fail(HSNF4_ERR_INVALID, "stream_prefetch_ahead: NULL streamer or list");
  for (int k = 0; k < n; ++k) {
    int rc = check_block("stream_prefetch_ahead", s, upcoming[k]);
    if (rc) return rc;
  }
  std::lock_guard<std::mutex> lk(s->mu);
  for (int k = 0; k < n; ++k) {
    const int b = upcoming[k];
    if (s->find(b, kLoaded) >= 0) continue;
    if (s->cfg.reuse_resident) {
      if (s->find(b, kAcquired) >= 0) continue;  // in use now and still resident then
      const int rel = s->find(b, kReleased);
      if (rel >= 0) {  // keep it: it is needed soon
        s->slots[rel].state = kLoaded;
        s->stats.reuses += 1;
        continue;
      }
    }
    if (!s->cfg.enable_prefetch) break;
    const int i = choose_slot(s, b, upcoming + k + 1, n - k - 1, /*quiet=*/true);
    if (i < 0) break;  // the ring is full of blocks still needed: stop here
    int rc = enqueue_copy(s, i, b, nullptr);
    if (rc) return rc;
    if (issued) ++*issued;
  }
  return HSNF4_OK;
}

int stream_block_acquire(hsnf4_streamer* s, int block, void* compute_stream,
                         hsnf4_nf4_weight* out, int max_out) {
  int rc = check_block("stream_block_acquire", s, block);
  if (rc) return rc;
  if (!out) return fail(HSNF4_ERR_INVALID, "stream_block_acquire: out is NULL");
  cudaStream_t cs = static_cast<cudaStream_t>(compute_stream);
  std::lock_guard<std::mutex> lk(s->mu);
  int need = 0;
  for (int l = s->first_layer(block); l < s->end_layer(block); ++l) need += s->layers[l].n_proj;
  if (max_out < need)
    return fail(HSNF4_ERR_INVALID, "stream_block_acquire: out holds %d weights, block needs %d",
                max_out, need);
  int i = s->find(block, kLoaded);
  if (i < 0 && s->cfg.reuse_resident) {
    if (s->find(block, kAcquired) >= 0)
      return fail(HSNF4_ERR_STATE, "stream_block_acquire: block %d is already acquired", block);
    i = s->find(block, kReleased);
  }
  if (i < 0) {
    if (s->cfg.enable_prefetch)
      return fail(HSNF4_ERR_STATE, "stream_block_acquire: block %d was not prefetched", block);
    i = choose_slot(s, block);
    if (i < 0) return HSNF4_ERR_STATE;
    rc = enqueue_copy(s, i, block, cs);
    if (rc) return rc;
  }
  Slot& sl = s->slots[i];
  rc = cuda_status(cudaStreamWaitEvent(cs, sl.ready, 0), "acquire: wait ready");
  if (rc) return rc;
  uint8_t* base = s->ring + static_cast<size_t>(i) * s->slot_bytes;
  int k = 0;
  for (int l = s->first_layer(block); l < s->end_layer(block); ++l) {
    const hsnf4_layer_desc& d = s->layers[l];
    const size_t lo = s->layer_off[l] - s->block_off(block);
    for (int p = 0; p < d.n_proj; ++p) {
      size_t co, ao;
      layer_offsets(d, p, &co, &ao);
      out[k].codes = base + lo + co;
      out[k].absmax = (d.base_format == HSNF4_BASE_BF16)
                          ? nullptr
                          : reinterpret_cast<const float*>(base + lo + ao);
      out[k].n_out = d.n_out[p];
      out[k].k_in = d.k_in[p];
      out[k].format = d.base_format;
      out[k].reserved = 0;
      ++k;
    }
  }
  sl.state = kAcquired;
  sl.last_use = ++s->seq;
  s->stats.acquires += 1;
  return HSNF4_OK;
}

int stream_block_acquire_host(hsnf4_streamer* s, int block, int timeout_ms) {
  int rc = check_block("stream_block_acquire_host", s, block);
  if (rc) return rc;
  cudaEvent_t ev;
  {
    std::lock_guard<std::mutex> lk(s->mu);
    int i = s->find(block, kLoaded);
    if (i < 0) i = s->find(block, kAcquired);
    if (i < 0)
      return fail(HSNF4_ERR_STATE, "stream_block_acquire_host: block %d was not prefetched",
                  block);
    ev = s->slots[i].ready;
  }
  const auto deadline =
      std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms < 0 ? 0 : timeout_ms);
  for (;;) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return HSNF4_OK;
    if (e != cudaErrorNotReady) return cuda_status(e, "stream_block_acquire_host: event query");
    if (std::chrono::steady_clock::now() >= deadline)
      return fail(HSNF4_ERR_TIMEOUT, "stream_block_acquire_host: block %d not ready after %d ms",
                  block, timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

int stream_block_release(hsnf4_streamer* s, int block, void* compute_stream) {
  int rc = check_block("stream_block_release", s, block);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(s->mu);
  const int i = s->find(block, kAcquired);
  if (i < 0)
    return fail(HSNF4_ERR_STATE, "stream_block_release: block %d is not acquired", block);
  Slot& sl = s->slots[i];
  rc = record(sl.free, static_cast<cudaStream_t>(compute_stream), "release: record free");
  if (rc) return rc;
  sl.free_recorded = true;
  sl.state = kReleased;
  s->stats.releases += 1;
  if (s->cfg.poison_on_release) {
    // debug: a read after release now sees 0xFF bytes instead of stale data
    rc = cuda_status(cudaStreamWaitEvent(s->copy, sl.free, 0), "release: poison wait");
    if (!rc)
      rc = cuda_status(cudaMemsetAsync(s->ring + static_cast<size_t>(i) * s->slot_bytes, 0xFF,
                                       s->slot_bytes, s->copy),
                       "release: poison memset");
    if (rc) return rc;
    sl.block = -1;
    sl.state = kEmpty;
  }
  return HSNF4_OK;
}

int stream_stats(const hsnf4_streamer* s, hsnf4_stream_stats* out) {
  if (!s || !out) return fail(HSNF4_ERR_INVALID, "stream_stats: NULL argument");
  *out = s->stats;
  return HSNF4_OK;
}

int stream_destroy(hsnf4_streamer* s) {
  if (!s) return HSNF4_OK;
  int rc = HSNF4_OK;
  if (s->copy || (!s->slots.empty() && s->slots[0].ready))
    rc = cuda_status(cudaStreamSynchronize(s->copy), "stream_destroy: synchronize copy stream");
  for (auto& sl : s->slots) {
    if (sl.ready) cudaEventDestroy(sl.ready);
    if (sl.free) cudaEventDestroy(sl.free);
  }
  delete s;
  return rc;
}

}  // extern "C"
