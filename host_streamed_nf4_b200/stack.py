"""A stack of NF4 LoRA layers driven through the C ABI, streamed or resident.

base="bf16" holds the frozen base as dense bf16 instead (the
quantization="bf16_bitwise" base of the Poros API reference: 3.56x the
bytes per weight, the same ring, no dequantization).

Each layer has the 7 LoRA-targeted projections of its model family.  The
frozen NF4 base of the whole stack lives in one pinned host slab (quantized
on the GPU, layer by layer, and copied down -- the bounded-residency load
the consumer-GPU page describes for its streamed loader); adapters,
activations, gradients and workspaces live in VRAM.

One step = forward through the layers in order, then backward in reverse
order (the backward needs every block's weights again).
  * streamed: blocks of `block_size` layers are fetched into the 2-slot
    ring, one block ahead on the copy stream; a block still resident at the
    forward/backward turn-around is reused unless `reuse_resident=False`.
  * resident: the whole slab is copied to VRAM once; the same kernels read
    the same bytes from there.

Inputs (synthetic, seeded): every layer sees the same activations -- X [T,
hidden] for q/k/v/gate/up, a [T, heads*head_dim] input for o, a [T, inter]
input for down -- and per-projection upstream gradients dY [T, n_out].  The
layers are not chained (no attention or MLP between them): what the path is
about is that weights arrive before their matmul and that streaming does
not change a single bit.
"""
from __future__ import annotations

import torch

from . import hsnf4, synth

INPUT_OF = {"q": "h", "k": "h", "v": "h", "o": "o", "gate": "h", "up": "h", "down": "i"}

# How a layer's 7 projections are batched into grouped launches.
#   decoder: what a decoder layer's data dependencies allow -- q/k/v share
#            their input, o needs attention, gate/up share their input, down
#            needs the MLP activation (the backward runs the groups reversed);
#   layer:   all 7 in one group (they are independent in this stack);
#   none:    one launch sequence per projection.
GROUPINGS = {
    "decoder": [[0, 1, 2], [3], [4, 5], [6]],
    "layer": [[0, 1, 2, 3, 4, 5, 6]],
    "none": [[0], [1], [2], [3], [4], [5], [6]],
}


def _randn_bf16(shape, std, gen, device):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(
        torch.bfloat16)


def _gen(device, seed, *keys):
    return torch.Generator(device=device).manual_seed(synth.sub_seed(seed, *keys) % (2**63))


class LayerStack:
    def __init__(self, family: synth.Family, n_layers: int, T: int, *, block_size: int = 4,
                 streamed: bool = True, reuse_resident: bool = True, enable_prefetch: bool = True,
                 poison_on_release: bool = False, r: int = synth.RANK, alpha: float = synth.ALPHA,
                 seed: int = 42, device=None, grouping: str = "layer", n_slots: int = 2,
                 base: str = "nf4", dropout: float = 0.0, data_seed=None, shard=None,
                 slab=None, shard_slab: bool = True):
        """shard = (rank, world, gather_factory): stream 1/world of every
        block (sharded stream); gather_factory(ring) returns the streamer's
        gather callback (dist.ring_gather).  data_seed: seed of the
        activations and upstream gradients (default: seed); the weights and
        adapters always come from seed, as data-parallel ranks share them.
        slab: an already filled pinned slab of a stack with the same family,
        layer count, base and seed (e.g. another stack's .slab), used as is
        instead of drawing and quantizing the base again.
        shard_slab (sharded streams): pin only this rank's shards of every
        block, about 1/world of the base, so that the ranks of a node hold
        one copy of it between them; False pins the whole base per rank."""
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        dev = self.device
        self.family, self.L, self.T, self.r, self.alpha = family, n_layers, T, r, alpha
        self.block_size, self.streamed = block_size, streamed
        self.projs = family.projections()
        self.P = len(self.projs)
        self.groups = GROUPINGS[grouping]
        if base not in ("nf4", "bf16"):
            raise ValueError(f"base must be 'nf4' or 'bf16' (got {base!r})")
        self.base = base
        self.base_format = hsnf4.BASE_BF16 if base == "bf16" else hsnf4.BASE_NF4
        # LoRA dropout on the adapter branch: the mask of (step, layer,
        # projection) is drawn from a counter-based generator, so the backward
        # re-draws exactly the forward's mask
        self.dropout, self.seed, self.step_idx = float(dropout), int(seed), 0
        self.desc = hsnf4.layer_desc([(n, k) for _, n, k in self.projs], self.base_format)
        self.descs = [self.desc] * n_layers
        self.layer_bytes = hsnf4.layer_bytes(self.desc)
        self.offs = [hsnf4.layer_offsets(self.desc, p) for p in range(self.P)]
        self.n_blocks = (n_layers + block_size - 1) // block_size
        self.shard_slab = bool(shard) and streamed and shard_slab
        if self.shard_slab:
            if slab is not None:
                raise ValueError("slab: a shard slab is filled by the stack itself")
            self.shard_layout, total = hsnf4.shard_slab_layout(self.descs, block_size, shard[1],
                                                               shard[0])
            self.slab = torch.empty(max(total, 1), dtype=torch.uint8, pin_memory=True)
            self._fill_shard_slab(seed, shard[0], shard[1])
        elif slab is not None:
            if slab.dtype != torch.uint8 or slab.numel() != hsnf4.slab_bytes(self.descs) or \
                    not slab.is_pinned():
                raise ValueError("slab: expected a pinned uint8 tensor of this stack's slab size")
            self.slab = slab
        else:
            self.slab = torch.empty(hsnf4.slab_bytes(self.descs), dtype=torch.uint8,
                                    pin_memory=True)
            self._fill_slab(seed)

        self.compute = torch.cuda.current_stream(dev)
        self.shard = shard
        if streamed:
            world = shard[1] if shard else 0
            self.ring = torch.empty(hsnf4.ring_bytes(self.descs, block_size, n_slots, world),
                                    dtype=torch.uint8, device=dev)
            self.copy_stream = torch.cuda.Stream(dev)
            sh = (shard[0], shard[1], shard[2](self.ring)) if shard else None
            self.streamer = hsnf4.Streamer(self.slab, self.descs, block_size, self.ring,
                                           self.copy_stream, enable_prefetch=enable_prefetch,
                                           reuse_resident=reuse_resident,
                                           poison_on_release=poison_on_release, n_slots=n_slots,
                                           shard=sh, shard_slab=self.shard_slab)
        else:
            self.dev_slab = self.slab.to(dev)
            self.streamer = None

        # activations and upstream gradients (shared by all layers)
        h, d = family.hidden, family.head_dim
        g = _gen(dev, seed if data_seed is None else data_seed, 1_000_001)
        self.X = {"h": _randn_bf16((T, h), 1.0, g, dev),
                  "o": _randn_bf16((T, family.heads * d), 1.0, g, dev),
                  "i": _randn_bf16((T, family.inter), 1.0, g, dev)}
        self.dY = [_randn_bf16((T, n), 1.0, g, dev) for _, n, _ in self.projs]
        # adapters (always resident) and per-(layer, projection) outputs kept for the backward
        # every adapter gradient lives in one flat fp32 buffer (dA then dB per
        # layer and projection), so that data-parallel ranks can sum them with
        # one all-reduce
        per_layer = sum(r * k + n * r for _, n, k in self.projs)
        self.grad_flat = torch.empty(n_layers * per_layer, dtype=torch.float32, device=dev)
        self.A, self.B, self.t, self.dA, self.dB = [], [], [], [], []
        off = 0
        for l in range(n_layers):
            ga = _gen(dev, seed, 2_000_000 + l)
            self.A.append([_randn_bf16((r, k), synth.A_STD, ga, dev) for _, _, k in self.projs])
            self.B.append([_randn_bf16((n, r), synth.B_STD, ga, dev) for _, n, _ in self.projs])
            self.t.append([torch.empty(T, r, dtype=torch.float32, device=dev) for _ in self.projs])
            dA, dB = [], []
            for _, n, k in self.projs:
                dA.append(self.grad_flat[off: off + r * k].view(r, k))
                off += r * k
                dB.append(self.grad_flat[off: off + n * r].view(n, r))
                off += n * r
            self.dA.append(dA)
            self.dB.append(dB)
        self.Y = [torch.empty(T, n, dtype=torch.bfloat16, device=dev) for _, n, _ in self.projs]
        self.dX = [torch.empty(T, k, dtype=torch.bfloat16, device=dev) for _, _, k in self.projs]
        # workspaces: the largest any group needs (addresses do not matter here)
        dummy = hsnf4.Nf4WeightC(0, 0, 0, 0)
        ws_f = ws_b = 256
        for grp in self.groups:
            fa = [hsnf4.FwdArgs(hsnf4.Nf4WeightC(0, 0, self.projs[p][1], self.projs[p][2]), 0, 0, 0,
                                0, 1, self.dropout) for p in grp]
            ba = [hsnf4.BwdArgs(hsnf4.Nf4WeightC(0, 0, self.projs[p][1], self.projs[p][2]),
                                0, 0, 0, 0, 0, 0, 0, 0, self.dropout) for p in grp]
            ws_f = max(ws_f, hsnf4.group_fwd_workspace_bytes(fa, T, r))
            ws_b = max(ws_b, hsnf4.group_bwd_workspace_bytes(ba, T, r))
        del dummy
        self.ws_f = torch.empty(ws_f, dtype=torch.uint8, device=dev)
        self.ws_b = torch.empty(ws_b, dtype=torch.uint8, device=dev)
        self._prefetched = False
        torch.cuda.synchronize(dev)

    # ------------------------------------------------------------------ setup

    def base_weight_bf16(self, l: int, p: int) -> torch.Tensor:
        """The seeded bf16 weight [n_out, k_in] of layer l, projection p that
        the slab holds (quantized, for an NF4 base), drawn again on the
        device: lets a checker quantize it independently."""
        _, n, k = self.projs[p]
        return _randn_bf16((n, k), synth.W_STD, _gen(self.device, self.seed, l, p), self.device)

    def _layer_into(self, buf: torch.Tensor, l: int, seed: int):
        """Write layer l's slab bytes (drawn and quantized on the device)
        into the device byte buffer buf [layer_bytes]."""
        dev = self.device
        for p, (_, n, k) in enumerate(self.projs):
            w = _randn_bf16((n, k), synth.W_STD, _gen(dev, seed, l, p), dev)
            co, ao = self.offs[p]
            if self.base_format == hsnf4.BASE_BF16:
                buf[co: co + n * k * 2].copy_(w.view(torch.uint8).flatten())
                continue
            W = hsnf4.nf4_quantize_pack(w)
            buf[co: co + n * k // 2].copy_(W.codes)
            buf[ao: ao + n * k // 16].copy_(W.absmax.view(torch.uint8))

    def _fill_shard_slab(self, seed: int, rank: int, world: int):
        """This rank's shard of every block, block after block: each block is
        built on the device and only the rank's byte range copied down."""
        dev = self.device
        block = torch.zeros(self.block_size * self.layer_bytes, dtype=torch.uint8, device=dev)
        for b in range(self.n_blocks):
            layers = list(self.block_layers(b))
            for i, l in enumerate(layers):
                self._layer_into(block[i * self.layer_bytes: (i + 1) * self.layer_bytes], l, seed)
            _, off, n = hsnf4.shard_range(len(layers) * self.layer_bytes, world, rank)
            at, n2 = self.shard_layout[b]
            assert n2 == n
            if n:
                self.slab[at: at + n].copy_(block[off: off + n])
        torch.cuda.synchronize(dev)
        del block

    def device_weight(self, l: int, p: int):
        """Layer l, projection p of the frozen base on the device, drawn and
        quantized again (independent of where the slab keeps it)."""
        w = self.base_weight_bf16(l, p)
        if self.base_format == hsnf4.BASE_BF16:
            return hsnf4.Bf16Weight(w)
        return hsnf4.nf4_quantize_pack(w)

    def pinned_bytes(self) -> int:
        """Page-locked host bytes this stack holds for the frozen base."""
        return self.slab.numel()

    def _fill_slab(self, seed: int):
        dev = self.device
        for l in range(self.L):
            base = l * self.layer_bytes
            for p, (_, n, k) in enumerate(self.projs):
                w = _randn_bf16((n, k), synth.W_STD, _gen(dev, seed, l, p), dev)
                co, ao = self.offs[p]
                if self.base_format == hsnf4.BASE_BF16:
                    self.slab[base + co: base + co + n * k * 2].copy_(w.view(torch.uint8).flatten())
                    del w
                    continue
                W = hsnf4.nf4_quantize_pack(w)
                self.slab[base + co: base + co + n * k // 2].copy_(W.codes)
                self.slab[base + ao: base + ao + n * k // 16].view(torch.float32).copy_(W.absmax)
                del w, W
        torch.cuda.synchronize(dev)

    def layer_weights(self, l: int):
        """Resident-mode weights of layer l (views into the device copy)."""
        base = l * self.layer_bytes
        out = []
        for p, (_, n, k) in enumerate(self.projs):
            co, ao = self.offs[p]
            if self.base_format == hsnf4.BASE_BF16:
                out.append(hsnf4.Nf4WeightC(self.dev_slab.data_ptr() + base + co, None, n, k,
                                            hsnf4.BASE_BF16, 0))
            else:
                out.append(hsnf4.Nf4WeightC(self.dev_slab.data_ptr() + base + co,
                                            self.dev_slab.data_ptr() + base + ao, n, k,
                                            hsnf4.BASE_NF4, 0))
        return out

    def block_layers(self, b: int):
        return range(b * self.block_size, min((b + 1) * self.block_size, self.L))

    # ------------------------------------------------------------------ passes

    def _weights(self, b: int):
        if self.streamed:
            return self.streamer.acquire(b, self.compute)
        ws = []
        for l in self.block_layers(b):
            ws += self.layer_weights(l)
        return ws

    def _release(self, b: int):
        if self.streamed:
            self.streamer.release(b, self.compute)

    def dropout_of(self, l: int, p: int):
        """(p, seed, offset) of layer l, projection p in the current step, or
        None: the offset packs (step, layer, projection)."""
        if self.dropout <= 0.0:
            return None
        return (self.dropout, self.seed, (self.step_idx << 32) | (l << 4) | p)

    def _fwd_block(self, ws, b, record):
        for i, l in enumerate(self.block_layers(b)):
            for grp in self.groups:
                args = [hsnf4.fwd_args(ws[i * self.P + p], self.X[INPUT_OF[self.projs[p][0]]],
                                       self.A[l][p], self.B[l][p], self.Y[p], self.t[l][p],
                                       self.dropout_of(l, p))
                        for p in grp]
                hsnf4.lora_group_fwd(args, self.T, self.r, self.alpha, self.ws_f,
                                     stream=self.compute)
                if record is not None:
                    for p in grp:
                        record(l, p, "Y", self.Y[p])

    def _bwd_block(self, ws, b, record):
        layers = list(self.block_layers(b))
        for i in reversed(range(len(layers))):
            l = layers[i]
            for grp in reversed(self.groups):
                args = [hsnf4.bwd_args(ws[i * self.P + p], self.X[INPUT_OF[self.projs[p][0]]],
                                       self.t[l][p], self.A[l][p], self.B[l][p], self.dY[p],
                                       self.dX[p], self.dA[l][p], self.dB[l][p],
                                       self.dropout_of(l, p))
                        for p in grp]
                hsnf4.lora_group_bwd(args, self.T, self.r, self.alpha, self.ws_b,
                                     stream=self.compute)
                if record is not None:
                    for p in grp:
                        record(l, p, "dX", self.dX[p])

    def forward(self, record=None):
        nb = self.n_blocks
        if self.streamed:
            self.streamer.prefetch(0)
        for b in range(nb):
            ws = self._weights(b)
            if self.streamed and b + 1 < nb:
                self.streamer.prefetch(b + 1)
            self._fwd_block(ws, b, record)
            self._release(b)

    def backward(self, record=None):
        nb = self.n_blocks
        if self.streamed:
            self.streamer.prefetch(nb - 1)
        for b in reversed(range(nb)):
            ws = self._weights(b)
            if self.streamed and b > 0:
                self.streamer.prefetch(b - 1)
            self._bwd_block(ws, b, record)
            self._release(b)

    def visits(self):
        """One step's block visits: forward in order, then backward reversed."""
        nb = self.n_blocks
        return [(b, True) for b in range(nb)] + [(b, False) for b in reversed(range(nb))]

    def step(self, record=None):
        """One training step.  Streamed: at each visit the block is acquired,
        the upcoming visits (wrapping into the next step) are prefetched as
        far as the ring allows, the block is computed and released."""
        V = self.visits()
        if not self.streamed:
            for b, fwd in V:
                ws = self._weights(b)
                (self._fwd_block if fwd else self._bwd_block)(ws, b, record)
            self.step_idx += 1
            return
        n = len(V)
        look = 2 * self.streamer.n_slots
        if not self._prefetched:
            self.streamer.prefetch_ahead([V[0][0]])
            self._prefetched = True
        for i, (b, fwd) in enumerate(V):
            ws = self.streamer.acquire(b, self.compute)
            self.streamer.prefetch_ahead([V[(i + j) % n][0] for j in range(1, look + 1)])
            (self._fwd_block if fwd else self._bwd_block)(ws, b, record)
            self.streamer.release(b, self.compute)
        self.step_idx += 1

    def step_single_block(self, record=None):
        """A one-block stack whose block is re-streamed every step: acquire the
        copy made during the previous step, start the next step's copy into the
        other slot, run forward and backward on the block, release it.  (Needs
        reuse_resident=False, so that the prefetch makes a fresh copy.)"""
        if not (self.streamed and self.n_blocks == 1):
            raise ValueError("step_single_block needs a streamed one-block stack")
        if not self._prefetched:
            self.streamer.prefetch(0)
            self._prefetched = True
        ws = self.streamer.acquire(0, self.compute)
        self.streamer.prefetch(0)
        self._fwd_block(ws, 0, record)
        self._bwd_block(ws, 0, record)
        self.streamer.release(0, self.compute)
        self.step_idx += 1

    # ------------------------------------------------------------------ checks

    def resident_check(self) -> dict:
        """Bitwise check of the last step against a resident recomputation:
        layers 0 and L-1 are run again from weights drawn and quantized
        afresh on the device (not from the ring), with the step's inputs, and
        their t, dA, dB -- plus Y of layer L-1 (the forward's last output)
        and dX of layer 0 (the backward's last output) -- must equal what
        the step left behind.  Call right after step(); returns the
        comparison per layer."""
        dev, T, r = self.device, self.T, self.r
        step = self.step_idx - 1  # the step whose outputs are checked
        out = {}
        for l in sorted({0, self.L - 1}):
            ws = [self.device_weight(l, p) for p in range(self.P)]
            Y = [torch.empty(T, n, dtype=torch.bfloat16, device=dev) for _, n, _ in self.projs]
            t = [torch.empty(T, r, dtype=torch.float32, device=dev) for _ in self.projs]
            dX = [torch.empty(T, k, dtype=torch.bfloat16, device=dev) for _, _, k in self.projs]
            dA = [torch.empty(r, k, dtype=torch.float32, device=dev) for _, _, k in self.projs]
            dB = [torch.empty(n, r, dtype=torch.float32, device=dev) for _, n, _ in self.projs]

            def drop(p, l=l):
                if self.dropout <= 0.0:
                    return None
                return (self.dropout, self.seed, (step << 32) | (l << 4) | p)

            for grp in self.groups:
                args = [hsnf4.fwd_args(ws[p], self.X[INPUT_OF[self.projs[p][0]]], self.A[l][p],
                                       self.B[l][p], Y[p], t[p], drop(p)) for p in grp]
                hsnf4.lora_group_fwd(args, T, r, self.alpha, self.ws_f, stream=self.compute)
            for grp in reversed(self.groups):
                args = [hsnf4.bwd_args(ws[p], self.X[INPUT_OF[self.projs[p][0]]], t[p],
                                       self.A[l][p], self.B[l][p], self.dY[p], dX[p], dA[p],
                                       dB[p], drop(p)) for p in grp]
                hsnf4.lora_group_bwd(args, T, r, self.alpha, self.ws_b, stream=self.compute)
            torch.cuda.synchronize(dev)
            eq = all(torch.equal(t[p], self.t[l][p]) and torch.equal(dA[p], self.dA[l][p]) and
                     torch.equal(dB[p], self.dB[l][p]) for p in range(self.P))
            if l == self.L - 1:
                eq = eq and all(torch.equal(Y[p], self.Y[p]) for p in range(self.P))
            if l == 0:
                eq = eq and all(torch.equal(dX[p], self.dX[p]) for p in range(self.P))
            out[l] = bool(eq)
            del ws, Y, t, dX, dA, dB
        return out

    # ------------------------------------------------------------------ accounting

    def block_bytes(self, b: int) -> int:
        return len(self.block_layers(b)) * self.layer_bytes

    def steady_h2d_bytes_per_step(self, reuse_resident: bool = True, n_slots: int = 2) -> int:
        """Bytes one steady-state step copies host -> device.  Without reuse
        every block crosses once per pass.  With reuse, the blocks still
        resident at each of the two turn-arounds (forward -> backward and
        backward -> next forward) are not copied again: the n_slots blocks
        nearest the turn-around."""
        nb = self.n_blocks
        total = 2 * sum(self.copied_bytes(b) for b in range(nb))
        if not reuse_resident:
            return total
        k = min(n_slots, nb)
        reused = sum(self.copied_bytes(nb - 1 - j) for j in range(k)) + \
            sum(self.copied_bytes(j) for j in range(k))
        return max(total - reused, 0)

    def copied_bytes(self, b: int) -> int:
        """Bytes this rank copies host -> device for block b: the whole block,
        or its shard of it in a sharded stream."""
        if not self.shard:
            return self.block_bytes(b)
        return hsnf4.shard_range(self.block_bytes(b), self.shard[1], self.shard[0])[2]

    def step_inputs(self):
        """The device tensors a step reads that come from outside (the
        activations and upstream gradients), for end-to-end timing."""
        return list(self.X.values()) + list(self.dY)

    def tokens_per_step(self) -> int:
        return self.T

    def close(self):
        if self.streamer is not None:
            self.streamer.close()
            self.streamer = None
