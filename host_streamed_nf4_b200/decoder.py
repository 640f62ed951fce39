"""A stack of full decoder layers on the streamed NF4 base, rematerialized
per block.

The pages train LoRA on Qwen2.5 / Llama-3.1 decoder layers, streaming each
block of layers in for the forward and again for the backward, where the
block's forward is recomputed so that activation memory is one block's
worth (Poros on consumer GPUs, "OOM playbook": activation memory at the
rematerialization boundary; Poros API reference, patch_hf_model: forward and
backward routed through per-block autograd functions).  Each layer is the
pre-norm decoder layer of those families around its seven LoRA projections:

    a = rmsnorm(h0)           q, k, v = lora(a)        att = sdpa(q, k, v)
    h1 = h0 + lora_o(att)     b = rmsnorm(h1)          m = silu(lora_gate(b)) lora_up(b)
    h2 = h1 + lora_down(m)

(causal grouped-query attention, head_dim 128, no rotary embedding).  The
forward keeps only each block's input; the backward of a block recomputes
its layers' forward from that input with the same weights (the block is in
its ring slot for the backward visit anyway) and the same dropout masks (the
counter-based generator is keyed by step, layer and projection), then runs
the layers' backward in reverse.  The last block is the exception: its
backward visit follows its forward visit at once, so its forward keeps
every layer's activations (the buffers a recompute would fill) and its
backward uses them as they are; the activation memory is still one block's.  Every step of the path runs in the
library's kernels; this module only sequences the calls and owns buffers.

Synthetic data: the stack's input h0 [T, hidden] and the gradient arriving
at its output are seeded normals; the norm gains are 1 + N(0, 0.1^2).
"""
from __future__ import annotations

import torch

from . import hsnf4, synth
from .stack import LayerStack, _gen, _randn_bf16

EPS = 1e-6
Q, K, V, O, GATE, UP, DOWN = range(7)


class DecoderStack(LayerStack):
    def __init__(self, family: synth.Family, n_layers: int, T: int, **kw):
        if family.head_dim != 128:
            raise ValueError("the attention kernels take head_dim 128")
        kw.setdefault("grouping", "decoder")
        if kw["grouping"] != "decoder":
            raise ValueError("a decoder layer runs its projections in decoder grouping")
        super().__init__(family, n_layers, T, **kw)
        dev, f = self.device, family
        h, I, H, KV, d = f.hidden, f.inter, f.heads, f.kv_heads, f.head_dim
        self.H, self.KV = H, KV
        seed = kw.get("seed", 42)
        data_seed = kw.get("data_seed") or seed
        g = _gen(dev, seed, 3_000_000)
        self.g1 = [(1.0 + 0.1 * torch.randn(h, generator=g, device=dev)).to(torch.bfloat16)
                   for _ in range(n_layers)]
        self.g2 = [(1.0 + 0.1 * torch.randn(h, generator=g, device=dev)).to(torch.bfloat16)
                   for _ in range(n_layers)]
        gd = _gen(dev, data_seed, 3_000_001)
        self.h_in = _randn_bf16((T, h), 1.0, gd, dev)      # stack input
        self.dh_top = _randn_bf16((T, h), 1.0, gd, dev)    # gradient at the stack output

        def bf(*shape):
            return torch.empty(*shape, dtype=torch.bfloat16, device=dev)

        bs = self.block_size
        # block inputs kept by the forward (the rematerialization boundary);
        # block 0's input is h_in itself
        self.saved = [None] + [bf(T, h) for _ in range(1, self.n_blocks)]
        # per-layer activations of the block being recomputed / run forward
        self.act = [{"a": bf(T, h), "q": bf(T, H * d), "k": bf(T, KV * d), "v": bf(T, KV * d),
                     "att": bf(T, H * d), "lse": torch.empty(H, T, dtype=torch.float32,
                                                             device=dev),
                     "o": bf(T, h), "h1": bf(T, h), "b": bf(T, h), "gate": bf(T, I),
                     "up": bf(T, I), "m": bf(T, I), "dn": bf(T, h), "h0": None}
                    for _ in range(bs)]
        self.h_cur = bf(T, h)  # running hidden state (forward output of the last layer)
        self.rec_out = [bf(T, h) for _ in range(max(bs, 2))]  # layer outputs inside a block
        self.dh_cur = None
        self._kept = None  # block whose forward activations are still in self.act
        # backward scratch, shared by the layers
        self.gs = {"dm": bf(T, I), "dgate": bf(T, I), "dup": bf(T, I), "db_g": bf(T, h),
                   "db_u": bf(T, h), "dh1": bf(T, h), "datt": bf(T, H * d), "dq": bf(T, H * d),
                   "dk": bf(T, KV * d), "dv": bf(T, KV * d), "da_q": bf(T, h), "da_k": bf(T, h),
                   "da_v": bf(T, h), "dh_a": bf(T, h), "dh_b": bf(T, h),
                   "scratch": torch.empty(hsnf4.attention_scratch_bytes(T, H), dtype=torch.uint8,
                                          device=dev)}
        torch.cuda.synchronize(dev)

    # ------------------------------------------------------------ one layer

    def _lora_fwd(self, ws, l, projs, inputs, outputs):
        args = [hsnf4.fwd_args(ws[p], x, self.A[l][p], self.B[l][p], y, self.t[l][p],
                               self.dropout_of(l, p))
                for p, x, y in zip(projs, inputs, outputs)]
        hsnf4.lora_group_fwd(args, self.T, self.r, self.alpha, self.ws_f, stream=self.compute)

    def _lora_bwd(self, ws, l, projs, inputs, dys, dxs):
        args = [hsnf4.bwd_args(ws[p], x, self.t[l][p], self.A[l][p], self.B[l][p], dy, dx,
                               self.dA[l][p], self.dB[l][p], self.dropout_of(l, p))
                for p, x, dy, dx in zip(projs, inputs, dys, dxs)]
        hsnf4.lora_group_bwd(args, self.T, self.r, self.alpha, self.ws_b, stream=self.compute)

    def layer_forward(self, w, l, h0, out, s):
        """out = layer l (weights w: its 7 projections) applied to h0; every
        activation of the layer lands in the buffer set s."""
        st = self.compute
        s["h0"] = h0  # the input stays alive (block input or a kept layer output)
        hsnf4.rmsnorm_fwd(s["h0"], self.g1[l], EPS, y=s["a"], stream=st)
        self._lora_fwd(w, l, (Q, K, V), (s["a"],) * 3, (s["q"], s["k"], s["v"]))
        hsnf4.attention_fwd(s["q"], s["k"], s["v"], self.H, self.KV, o=s["att"], lse=s["lse"],
                            stream=st)
        self._lora_fwd(w, l, (O,), (s["att"],), (s["o"],))
        hsnf4.rmsnorm_fwd(s["h0"], self.g2[l], EPS, res=s["o"], h_out=s["h1"], y=s["b"],
                          stream=st)
        self._lora_fwd(w, l, (GATE, UP), (s["b"],) * 2, (s["gate"], s["up"]))
        hsnf4.swiglu_fwd(s["gate"], s["up"], m=s["m"], stream=st)
        self._lora_fwd(w, l, (DOWN,), (s["m"],), (s["dn"],))
        hsnf4.add(s["h1"], s["dn"], out=out, stream=st)

    def layer_backward(self, w, l, s, dh2, dh0):
        """dh0 = d(loss)/d(layer input) from dh2, with the activations s of a
        forward of this layer; accumulates nothing (dA, dB are overwritten)."""
        st, gs = self.compute, self.gs
        self._lora_bwd(w, l, (DOWN,), (s["m"],), (dh2,), (gs["dm"],))
        hsnf4.swiglu_bwd(s["gate"], s["up"], gs["dm"], da=gs["dgate"], db=gs["dup"], stream=st)
        self._lora_bwd(w, l, (GATE, UP), (s["b"],) * 2, (gs["dgate"], gs["dup"]),
                       (gs["db_g"], gs["db_u"]))
        hsnf4.rmsnorm_bwd(s["h1"], self.g2[l], (gs["db_g"], gs["db_u"]), EPS, dres=dh2,
                          dx=gs["dh1"], stream=st)
        self._lora_bwd(w, l, (O,), (s["att"],), (gs["dh1"],), (gs["datt"],))
        hsnf4.attention_bwd(s["q"], s["k"], s["v"], s["att"], s["lse"], gs["datt"], self.H,
                            self.KV, dq=gs["dq"], dk=gs["dk"], dv=gs["dv"], scratch=gs["scratch"],
                            stream=st)
        self._lora_bwd(w, l, (Q, K, V), (s["a"],) * 3, (gs["dq"], gs["dk"], gs["dv"]),
                       (gs["da_q"], gs["da_k"], gs["da_v"]))
        hsnf4.rmsnorm_bwd(s["h0"], self.g1[l], (gs["da_q"], gs["da_k"], gs["da_v"]), EPS,
                          dres=gs["dh1"], dx=dh0, stream=st)

    # ------------------------------------------------------------ blocks

    def block_input(self, b: int) -> torch.Tensor:
        return self.h_in if b == 0 else self.saved[b]

    def _fwd_block(self, ws, b, record):
        """Forward through block b from its input; the last layer writes the
        next block's saved input (the rematerialization boundary), the others
        ping-pong between two buffers: nothing else is kept.  The stack's last
        block instead keeps each layer's activations and outputs, for the
        backward visit that comes next."""
        layers = list(self.block_layers(b))
        keep = b == self.n_blocks - 1
        h = self.block_input(b)
        for i, l in enumerate(layers):
            last = i == len(layers) - 1
            if keep:
                out, s = (self.h_cur if last else self.rec_out[i]), self.act[i]
            elif last:
                out, s = self.saved[b + 1], self.act[0]
            else:
                out, s = (self.rec_out[i % 2] if self.block_size > 1 else self.h_cur), self.act[0]
            self.layer_forward(ws[i * self.P:(i + 1) * self.P], l, h, out, s)
            if record is not None:
                record(l, -1, "h_out", out)
            h = out
        self._kept = b if keep else None

    def _bwd_block(self, ws, b, record):
        """Recompute block b's forward from its saved input, keeping every
        layer's activations (unless its forward kept them), then
        back-propagate through its layers."""
        layers = list(self.block_layers(b))
        if self._kept == b:
            self._kept = None  # the forward just left these activations in self.act
        else:
            h = self.block_input(b)
            for i, l in enumerate(layers):
                out = self.rec_out[i]
                self.layer_forward(ws[i * self.P:(i + 1) * self.P], l, h, out, self.act[i])
                if record is not None:
                    record(l, -1, "h_out_recomputed", out)
                h = out
        if b == self.n_blocks - 1:
            self.dh_cur = self.dh_top  # gradient arriving at the stack output
        for i in reversed(range(len(layers))):
            l = layers[i]
            nxt = self.gs["dh_b"] if self.dh_cur is self.gs["dh_a"] else self.gs["dh_a"]
            self.layer_backward(ws[i * self.P:(i + 1) * self.P], l, self.act[i], self.dh_cur,
                                nxt)
            if record is not None:
                record(l, -1, "dh_in", nxt)
            self.dh_cur = nxt

    def step_inputs(self):
        return [self.h_in, self.dh_top]
