"""Layer-streamed LoRA training step over a frozen NF4 (or bf16) base.

The Soup pages' method ("how layer streaming works"): the frozen base is cut
into per-layer shards held in pinned host RAM; a ring of `stream_buffers`
(2..8) device slots is filled by a dedicated copy stream while the compute
stream works on the previous layer; the vocab-sized embed_tokens / lm_head
share one slot; every layer is read once for the forward pass and once more
for the checkpoint-recompute backward (layers still resident in the ring at
the turn-around are not copied again); only the LoRA adapters, their
gradients and their AdamW state live in VRAM permanently.

With ``stream_source="disk"`` (the pages' disk tier) the per-layer shards are
files instead, read ahead into ``read_ahead`` page-locked staging buffers by
the library's shard reader and copied from there.

This module is host-side orchestration only: device memory comes from
PyTorch, and every operation of the step (NF4 quantisation of the shards,
embedding, the decoder layers forward and backward, the chunked output head,
the losses and the AdamW update) runs in the CUDA library through its C ABI
(``_lib``).
"""
from __future__ import annotations

import os
import zlib
from dataclasses import dataclass

import torch

from . import _lib as L
from . import dp

ITEM_EMBED, ITEM_HEAD = L.SOUP_ITEM_EMBED, L.SOUP_ITEM_HEAD
PROJS = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass(frozen=True)
class ModelConfig:
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    rank: int
    alpha: float
    vocab: int
    n_layers: int
    eps: float = 1e-5
    theta: float = 5e5
    kind: str = "nf4"      # "nf4" or "bf16" frozen base
    tied: bool = False     # lm_head == embed_tokens

    @property
    def qkv_out(self):
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def o_in(self):
        return self.n_q_heads * self.head_dim

    def layer_cfg(self, prompt_share: int = 0) -> L.LayerCfg:
        """The layer calls' configuration; prompt_share > 0: pairs of
        sequences share their first prompt_share tokens, stored once."""
        return L.LayerCfg(self.hidden, self.n_q_heads, self.n_kv_heads, self.head_dim, self.intermediate,
                          self.rank, float(self.alpha), float(self.eps), float(self.theta),
                          2 if prompt_share else 0, int(prompt_share))

    @property
    def weight_kind(self):
        return L.SOUP_WEIGHT_NF4 if self.kind == "nf4" else L.SOUP_WEIGHT_BF16


def _seed(*parts) -> int:
    return zlib.crc32("/".join(str(p) for p in parts).encode()) & 0x7FFFFFFF


def _randn(shape, seed, std=1.0, mean=0.0):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


class SyntheticWeights:
    """Seeded synthetic frozen base drawn on the device: projections N(0, 0.02),
    RMSNorm weights 1 + 0.02 N(0, 1), embeddings N(0, 0.02)."""

    def __init__(self, cfg: ModelConfig, seed: int = 0, std: float = 0.02):
        self.cfg, self.seed, self.std = cfg, seed, std

    def layer(self, l):
        c = self.cfg
        shapes = {"qkv": (c.qkv_out, c.hidden), "o": (c.hidden, c.o_in), "gate_up": (2 * c.intermediate, c.hidden),
                  "down": (c.hidden, c.intermediate)}
        out = {k: _randn(s, _seed(self.seed, l, k), self.std) for k, s in shapes.items()}
        out["norm1"] = _randn((c.hidden,), _seed(self.seed, l, "norm1"), 0.02, 1.0).to(torch.bfloat16)
        out["norm2"] = _randn((c.hidden,), _seed(self.seed, l, "norm2"), 0.02, 1.0).to(torch.bfloat16)
        return out

    def vocab(self, which):
        c = self.cfg
        return _randn((c.vocab, c.hidden), _seed(self.seed, which), self.std).to(torch.bfloat16)

    def final_norm(self):
        return _randn((self.cfg.hidden,), _seed(self.seed, "final_norm"), 0.02, 1.0).to(torch.bfloat16)

    def lora(self, l):
        c = self.cfg
        r = c.rank
        shapes = {"A_qkv": (3 * r, c.hidden), "B_qkv": (c.qkv_out, r), "A_o": (r, c.o_in), "B_o": (c.hidden, r),
                  "A_gu": (2 * r, c.hidden), "B_gu": (2 * c.intermediate, r), "A_down": (r, c.intermediate),
                  "B_down": (c.hidden, r)}
        return {k: _randn(s, _seed(self.seed, l, k), 0.02).to(torch.bfloat16) for k, s in shapes.items()}


@dataclass(frozen=True)
class AdamW:
    """AdamW hyperparameters for the adapters.  The Soup pages' run sets only
    the learning rate (5e-4); the rest are the defaults of the Trainer those
    pages run on (betas 0.9 / 0.999, eps 1e-8, no weight decay)."""
    lr: float = 5e-4
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0


def token_rows(batch: int, seq: int, prompt_share: int = 0) -> int:
    """Token rows of `batch` sequences of `seq` tokens; with prompt_share,
    pairs share their first prompt_share tokens, stored once."""
    if not prompt_share:
        return batch * seq
    return (batch // 2) * (prompt_share + 2 * (seq - prompt_share))


def prompt_dedup_indices(batch: int, seq: int, prompt: int):
    """Index arrays (int32 numpy) of the shared-prompt layout of a preference
    batch (rows 2p chosen, 2p+1 rejected, sharing their first `prompt`
    tokens; the pair's token rows are [prompt | chosen continuation |
    rejected continuation]):
      phys      [token rows]: each token row's position in the flat ids [batch * seq]
                (prompt rows: the chosen sequence's);
      head_rows [batch * (seq - prompt + 1)]: for each sequence v and
                j = 0 .. seq - prompt, the token row of position prompt - 1 + j
                (the positions whose next-token log-probs cover the continuation);
      head_ids  [same]: the flat ids position of that (v, position);
      start, src: for each token row d, the head rows reading it are
                src[start[d]:start[d + 1]] (in increasing order)."""
    import numpy as np
    Lp, Lc = prompt, seq - prompt
    span = Lp + 2 * Lc

    def row(v, t):
        p, i = divmod(v, 2)
        return p * span + (t if t < Lp else Lp + i * Lc + (t - Lp))

    T = (batch // 2) * span
    phys = np.empty(T, np.int32)
    for v in range(batch):
        for t in range(seq):
            if v % 2 == 0 or t >= Lp:
                phys[row(v, t)] = v * seq + t
    hl = Lc + 1
    head_rows = np.array([row(v, Lp - 1 + j) for v in range(batch) for j in range(hl)], np.int32)
    head_ids = np.array([v * seq + Lp - 1 + j for v in range(batch) for j in range(hl)], np.int32)
    readers = [[] for _ in range(T)]
    for h, d in enumerate(head_rows):
        readers[d].append(h)
    start = np.zeros(T + 1, np.int32)
    start[1:] = np.cumsum([len(r) for r in readers])
    src = np.array([h for r in readers for h in r], np.int32)
    return phys, head_rows, head_ids, start, src


def device_bytes_lower_bound(cfg: ModelConfig, batch: int, seq: int, n_buffers: int, head_chunk: int,
                             prompt_share: int = 0) -> int:
    """Device bytes a streamed model needs at least, from the library's host
    size queries: the slot arena (n_buffers layer blobs + the vocab slot),
    the layer checkpoints [L+1, T, H] bf16, the layer workspace (which the
    head's shares when it is the larger), and the library's module-static
    device arrays."""
    lcfg = cfg.layer_cfg(prompt_share)
    blob = L.soup_layer_blob_bytes(lcfg, cfg.weight_kind)
    vocab = (cfg.vocab * cfg.hidden * 2 + 255) // 256 * 256
    T = token_rows(batch, seq, prompt_share)
    head_seq = seq - prompt_share + 1 if prompt_share else seq
    return (n_buffers * blob + vocab + (cfg.n_layers + 1) * T * cfg.hidden * 2 +
            max(L.soup_decoder_layer_workspace(lcfg, batch, seq),
                L.soup_head_workspace(cfg.vocab, cfg.hidden, batch, head_seq, head_chunk)) + L.static_device_bytes())


def precheck_device_bytes(cfg, batch, seq, n_buffers, head_chunk, cap, prompt_share=0):
    """Refuses, before any shard is built or any device memory is taken, a
    model whose lower-bound device need exceeds the cap (the stream plan makes
    the exact check once the model's own allocations are known)."""
    if not cap:
        return
    need = device_bytes_lower_bound(cfg, batch, seq, n_buffers, head_chunk, prompt_share)
    if need > cap:
        raise ValueError(f"the streamed model needs at least {need} device bytes ({n_buffers} slots, the vocab slot, "
                         f"checkpoints and workspaces) > device cap {cap}")


def kept_layer_count(n_layers: int, per_layer: int, arena: int, reserve: int, cap: int) -> int:
    """How many layers' q|k|v (per_layer bytes each) can be kept while
    soup_stream_plan still admits the model: arena (slots + vocab slot) +
    reserve + kept <= cap; all layers without a cap."""
    if per_layer <= 0:
        return 0
    if not cap:
        return n_layers
    room = cap - arena - reserve
    return max(0, min(n_layers, room // per_layer))


STREAM_RECOMPUTE = ("auto", "recompute", "keep")


def plan_keep(n_layers: int, qkv_bytes: int, saved_bytes: int, arena: int, reserve: int, cap: int,
              mode: str = "auto") -> list:
    """Per-layer plan of what the forward pass keeps for the backward (the
    pages' `stream_recompute` key): "saved" (every intermediate: no forward
    recompute in the backward), "qkv" (q|k|v only: the backward skips its
    q|k|v GEMM) or None (full recompute), such that the slot arena, the
    model's own device bytes (reserve) and the kept bytes fit a nonzero cap.

    recompute: keep nothing.  keep: every layer saved, or ValueError when
    that does not fit.  auto: q|k|v first for as many layers as fit (it saves
    the most recompute time per byte), then, when every layer keeps q|k|v
    and room is left, upgrade layers (from the first) to saved ones."""
    if mode not in STREAM_RECOMPUTE:
        raise ValueError(f"stream_recompute must be one of {STREAM_RECOMPUTE}, not {mode!r}")
    if mode == "recompute" or n_layers <= 0:
        return [None] * max(0, n_layers)
    room = (cap - arena - reserve) if cap else None
    if mode == "keep":
        need = n_layers * saved_bytes
        if room is not None and need > room:
            raise ValueError(f"stream_recompute='keep' needs {need} device bytes for {n_layers} saved layers, "
                             f"{max(0, room)} left under the device cap {cap}")
        return ["saved"] * n_layers
    if room is None:
        return ["saved"] * n_layers
    n_qkv = 0 if qkv_bytes <= 0 else max(0, min(n_layers, room // qkv_bytes))
    plan = ["qkv"] * n_qkv + [None] * (n_layers - n_qkv)
    if n_qkv == n_layers and saved_bytes > qkv_bytes:
        extra = room - n_layers * qkv_bytes
        for l in range(min(n_layers, max(0, extra) // (saved_bytes - qkv_bytes))):
            plan[l] = "saved"
    return plan


class StreamedLoRAModel:
    """Frozen base in pinned host blobs + a soup_plan slot ring + resident LoRA.

    weights: an object with ``layer(l)`` (fused fp32 device matrices qkv, o,
    gate_up, down and bf16 norm1/norm2), ``vocab(name)`` (bf16 [V, H]),
    ``final_norm()`` and ``lora(l)`` (bf16 fused LoRA factors).
    """

    def __init__(self, cfg: ModelConfig, batch: int, seq: int, n_buffers: int = 2, device_cap_bytes: int = 0,
                 head_chunk="auto", weights=None, seed: int = 0, adamw: AdamW | None = None,
                 task: str = "sft", stream_source: str = "ram", shard_dir: str | None = None,
                 read_ahead: int = 2, io_threads: int = 4, stream_recompute: str = "auto", prompt_dedup: int = 0):
        self.cfg, self.batch, self.seq, self.n_buffers = cfg, batch, seq, n_buffers
        if stream_source not in ("ram", "disk"):
            raise ValueError(f"stream_source must be 'ram' or 'disk', not {stream_source!r}")
        if stream_source == "disk" and not shard_dir:
            raise ValueError("stream_source='disk' needs a shard_dir for the per-layer shard files")
        self.stream_source, self.shard_dir = stream_source, shard_dir
        if stream_recompute not in STREAM_RECOMPUTE:
            raise ValueError(f"stream_recompute must be one of {STREAM_RECOMPUTE}, not {stream_recompute!r}")
        self.stream_recompute = stream_recompute
        self.disk = None
        self.adamw = adamw or AdamW()
        if task not in ("sft", "dpo", "simpo", "orpo"):
            raise ValueError(f"task must be 'sft', 'dpo', 'simpo' or 'orpo', not {task!r}")
        self.task = task
        # preference pairs with one prompt: the prompt's tokens are stored and
        # computed once per pair (prompt_dedup = the shared prompt length)
        if prompt_dedup:
            if task not in ("dpo", "simpo", "orpo"):
                raise ValueError("prompt_dedup applies to the preference tasks (pairs sharing a prompt)")
            if batch % 2 or not (0 < prompt_dedup < seq) or prompt_dedup % 128:
                raise ValueError(f"prompt_dedup needs an even batch and a shared prompt that is a positive multiple "
                                 f"of 128 shorter than the sequence (batch {batch}, prompt {prompt_dedup}, seq {seq})")
        self.prompt_dedup = int(prompt_dedup)
        self.T = token_rows(batch, seq, self.prompt_dedup)
        # the output head reads, per sequence, head_seq consecutive positions
        # (with a shared prompt: the last prompt position and the continuation)
        self.head_seq = seq - self.prompt_dedup + 1 if self.prompt_dedup else seq
        self.lcfg = cfg.layer_cfg(self.prompt_dedup)
        if head_chunk == "auto":
            # the most token rows per head chunk whose workspace still fits in
            # the layer workspace (which it shares): fewer, larger logits and
            # dx GEMMs at no extra device memory
            lw = L.soup_decoder_layer_workspace(self.lcfg, batch, seq)
            head_chunk = next((c for c in (1024, 512, 256) if
                               L.soup_head_workspace(cfg.vocab, cfg.hidden, batch, self.head_seq, c) <= lw), 128)
        self.head_chunk = int(head_chunk)
        precheck_device_bytes(cfg, batch, seq, n_buffers, self.head_chunk, device_cap_bytes, self.prompt_dedup)
        weights = weights or SyntheticWeights(cfg, seed)
        # the model's resident tensors first, the shard build's temporaries
        # after them: freed temporaries then leave whole cached segments that
        # empty_cache() can hand back (no resident tensor pins them)
        self._alloc(weights)
        self._build_blobs(weights)
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        # what each layer's forward pass keeps for its backward (identical
        # results either way): every intermediate ("saved": no recompute),
        # q|k|v ("qkv": the backward skips its q|k|v GEMM) or nothing, as the
        # device cap admits (stream_recompute)
        per = L.soup_decoder_layer_keep_bytes(self.lcfg, batch, seq)
        per_saved = L.soup_decoder_layer_saved_bytes(self.lcfg, batch, seq)
        self.keep_plan = plan_keep(cfg.n_layers, per, per_saved, self.n_buffers * self.blob_bytes + self.vocab_bytes,
                                   self.reserve_bytes, device_cap_bytes, stream_recompute)
        n_keep = sum(1 for k in self.keep_plan if k == "qkv")
        n_saved = sum(1 for k in self.keep_plan if k == "saved")
        self.keep, self.saved = None, None
        self.keep_row, self.saved_row = {}, {}
        if n_keep:
            self.keep = torch.empty((n_keep, per // 2), dtype=torch.float16, device="cuda")
            self.reserve_bytes += n_keep * per
        if n_saved:
            self.saved = torch.empty((n_saved, per_saved), dtype=torch.uint8, device="cuda")
            self.reserve_bytes += n_saved * per_saved
        for l, k in enumerate(self.keep_plan):
            if k == "qkv":
                self.keep_row[l] = len(self.keep_row)
            elif k == "saved":
                self.saved_row[l] = len(self.saved_row)
        self.plan = L.Plan(self.host_layers, self.blob_bytes, n_buffers, self.vocab_bytes, self.host_embed,
                           self.host_head, device_cap_bytes, self.reserve_bytes, n_layers=cfg.n_layers)
        if stream_source == "disk":
            # the pages' disk tier: shards read ahead from files into
            # read_ahead page-locked staging buffers along the step's visit
            # order (forward 0..L-1, backward L-1..0; a task="dpo" model's
            # shared visits follow the same order)
            self.disk = L.Disk(self.shard_paths, self.blob_bytes, read_ahead=read_ahead, n_slots=n_buffers,
                               io_threads=io_threads, pinned=True, direct=True)
            nl = cfg.n_layers
            self.disk.schedule(list(range(nl)) + list(range(nl - 1, -1, -1)))
        self._views = {}
        # When set to a dict, the backward pass stores dL/d(layer input) of
        # every layer in it (index l = input of layer l, n_layers = head output).
        self.capture_dh = None
        # the shard build's temporaries (fp32 weights, the staging blob) are
        # freed; hand their cached blocks back so that the device holds what
        # the model uses, not what building it once needed
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    # ------------------------------------------------------------ shard build
    def _build_blobs(self, weights):
        cfg = self.cfg
        kind = cfg.weight_kind
        self.blob_bytes = L.soup_layer_blob_bytes(self.lcfg, kind)
        staging = torch.empty(self.blob_bytes, dtype=torch.uint8, device="cuda")
        base = staging.data_ptr()
        v = L.soup_layer_blob_views(self.lcfg, kind, base)
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = torch.cuda.current_stream()

        def region(ptr, nbytes):
            off = ptr - base
            return staging[off:off + nbytes]

        disk = self.stream_source == "disk"
        self.host_layers = None if disk else []
        self.shard_paths = []
        if disk:
            os.makedirs(self.shard_dir, exist_ok=True)
            hb = torch.empty(self.blob_bytes, dtype=torch.uint8, pin_memory=True)
        for l in range(cfg.n_layers):
            w = weights.layer(l)
            for name in ("qkv", "o", "gate_up", "down"):
                sw = getattr(v, name)
                W = w[name].contiguous()
                assert tuple(W.shape) == (sw.out_features, sw.in_features), (name, W.shape)
                n = W.numel()
                if kind == L.SOUP_WEIGHT_NF4:
                    st_ = L.lib().soup_nf4_quantize(L.c_void_p(W.data_ptr()), sw.out_features, sw.in_features,
                                                    L.c_void_p(sw.codes), L.c_void_p(sw.absmax),
                                                    L.c_void_p(flag.data_ptr()), L.c_void_p(st.cuda_stream))
                    L._check("soup_nf4_quantize", st_)
                else:
                    region(sw.w, n * 2).view(torch.bfloat16).copy_(W.reshape(-1).to(torch.bfloat16))
            region(v.norm1, cfg.hidden * 2).view(torch.bfloat16).copy_(w["norm1"].reshape(-1))
            region(v.norm2, cfg.hidden * 2).view(torch.bfloat16).copy_(w["norm2"].reshape(-1))
            if disk:  # one shard file per layer, the blob's bytes
                hb.copy_(staging)
                path = os.path.join(self.shard_dir, f"layer_{l:03d}.bin")
                hb.numpy().tofile(path)
                self.shard_paths.append(path)
            else:
                hb = torch.empty(self.blob_bytes, dtype=torch.uint8, pin_memory=True)
                hb.copy_(staging)
                self.host_layers.append(hb)
            del w
        del staging
        V, H = cfg.vocab, cfg.hidden
        self.vocab_bytes = (V * H * 2 + 255) // 256 * 256

        def pin_vocab(t):
            hb = torch.zeros(self.vocab_bytes, dtype=torch.uint8, pin_memory=True)
            hb[:V * H * 2].copy_(t.reshape(-1).view(torch.uint8))
            return hb

        self.host_embed = pin_vocab(weights.vocab("embed"))
        self.host_head = self.host_embed if cfg.tied else pin_vocab(weights.vocab("lm_head"))
        torch.cuda.synchronize()

    # ------------------------------------------------------------ device state
    def _alloc(self, weights):
        cfg, T = self.cfg, self.T
        before = torch.cuda.memory_allocated()
        self.final_norm = weights.final_norm().contiguous()
        # LoRA factors (bf16, what the GEMMs read), their gradients (fp32),
        # and the AdamW state (fp32 master copy, first and second moments):
        # five flat buffers with one layout, each factor a view, so that the
        # data-parallel exchange is one all-reduce and the optimiser step one
        # launch over the whole adapter set (see dp.py)
        init = [weights.lora(l) for l in range(cfg.n_layers)]
        keys = [list(lo.keys()) for lo in init]
        shapes = [lo[k].shape for lo, ks in zip(init, keys) for k in ks]
        self.lora_flat, lviews = dp.flat_views(shapes, "cuda", torch.bfloat16)
        it = iter(lviews)
        self.lora = [{k: next(it) for k in ks} for ks in keys]
        for lo, src in zip(self.lora, init):
            for k, v in lo.items():
                v.copy_(src[k])
        del init
        self.grad_flat, views = dp.flat_views(shapes, "cuda")
        it = iter(views)
        self.grads = [{"d" + k: next(it) for k in ks} for ks in keys]
        self.master_flat = self.lora_flat.float()
        self.adam_m = torch.zeros_like(self.grad_flat)
        self.adam_v = torch.zeros_like(self.grad_flat)
        self.adam_t = 0
        self.nonfinite = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.lora_s = [L.layer_lora(lo) for lo in self.lora]
        self.grads_s = [L.layer_grads(g) for g in self.grads]
        self.ckpt = torch.empty((cfg.n_layers + 1, T, cfg.hidden), dtype=torch.bfloat16, device="cuda")
        self.dh = torch.empty((T, cfg.hidden), dtype=torch.float32, device="cuda")
        self.ws = torch.empty(L.soup_decoder_layer_workspace(self.lcfg, self.batch, self.seq), dtype=torch.uint8,
                              device="cuda")
        # the output head runs between the layer passes, never during a layer
        # call: its workspace shares the layer workspace's memory
        head_bytes = L.soup_head_workspace(cfg.vocab, cfg.hidden, self.batch, self.head_seq, self.head_chunk)
        if head_bytes <= self.ws.numel():
            self.head_ws = self.ws[:head_bytes]
        else:
            self.head_ws = torch.empty(head_bytes, dtype=torch.uint8, device="cuda")
        self.logp = torch.empty((self.batch, self.head_seq - 1), dtype=torch.float32, device="cuda")
        self.logp_ref = torch.empty_like(self.logp)
        self.coef = torch.empty_like(self.logp)
        self.loss = torch.zeros(1, dtype=torch.float32, device="cuda")
        self.seq_sums = torch.zeros(4 * max(1, self.batch // 2), dtype=torch.float32, device="cuda")
        self.ids = torch.empty((self.batch, self.seq), dtype=torch.int32, device="cuda")
        self.ids_tok = self.ids  # ids of the token rows (the shared-prompt layout: gathered)
        self.ids_head = self.ids  # targets of the rows the head reads
        if self.prompt_dedup:
            phys, hrows, hids, start, src = prompt_dedup_indices(self.batch, self.seq, self.prompt_dedup)
            dev = lambda a: torch.from_numpy(a).to("cuda")
            self.dd_phys, self.dd_head_rows, self.dd_head_ids = dev(phys), dev(hrows), dev(hids)
            self.dd_start, self.dd_src = dev(start), dev(src)
            self.ids_tok = torch.empty(self.T, dtype=torch.int32, device="cuda")
            self.ids_head = torch.empty((self.batch, self.head_seq), dtype=torch.int32, device="cuda")
            self.h_head = torch.empty((self.batch * self.head_seq, cfg.hidden), dtype=torch.bfloat16, device="cuda")
            self.dh_head = torch.empty((self.batch * self.head_seq, cfg.hidden), dtype=torch.float32, device="cuda")
        # DPO: running hidden state of the adapters-off reference pass, which
        # shares each layer visit with the policy's forward pass (ping-pong)
        self.h_ref = None
        if self.task == "dpo":
            self.h_ref = torch.empty((2, T, cfg.hidden), dtype=torch.bfloat16, device="cuda")
        # what the model holds besides the slot arena: its own tensors and the
        # library's module-static device arrays (held on every device that
        # loads the library, outside torch's allocator)
        self.reserve_bytes = torch.cuda.memory_allocated() - before + L.static_device_bytes()

    def views(self, base: int) -> L.LayerWeights:
        w = self._views.get(base)
        if w is None:
            w = L.soup_layer_blob_views(self.lcfg, self.cfg.weight_kind, base)
            self._views[base] = w
        return w

    @property
    def head_item(self):
        return ITEM_EMBED if self.cfg.tied else ITEM_HEAD

    # ------------------------------------------------------------ passes
    def _embed(self):
        """ckpt[0] = embed_tokens[ids].  The gather reads its rows straight
        from the pinned host matrix (mapped into the device address space), so
        only the batch's rows cross the host link, not the whole vocab matrix;
        the vocab slot is left to the lm_head."""
        L.soup_embed(self.host_embed.data_ptr(), self.cfg.vocab, self.cfg.hidden, self.ids_tok, self.T, self.ckpt[0])

    def _prefetch(self, l):
        """Brings layer l into a slot: from its pinned host blob, or with the
        disk tier from the reader's staging buffer (a layer still resident in
        a slot makes no copy either way)."""
        if self.disk is None or self.plan.resident(l):
            self.plan.prefetch(l)
            return
        host, ev = self.disk.acquire(l)
        try:
            self.plan.prefetch_from(l, host, ev)
        finally:
            self.disk.release(l)

    def _forward_layers(self, adapters_on: bool):
        """ckpt[0] -> ckpt[L], saving every layer input (the checkpoints)."""
        P, N, nl = self.plan, self.n_buffers, self.cfg.n_layers
        for l in range(min(N, nl)):
            self._prefetch(l)
        for l in range(nl):
            base = P.wait(l)
            if adapters_on:
                self._policy_fwd(l, self.views(base))
            else:
                L.soup_decoder_layer_fwd(self.views(base), self.lora_s[l], self.lcfg, self.ckpt[l], self.batch,
                                         self.seq, self.ckpt[l + 1], adapters_on, self.ws)
            P.release(l)
            if l + N < nl:
                self._prefetch(l + N)

    def _forward_layers_shared(self):
        """One visit per layer serves both forward passes of a DPO step: the
        reference (adapters off) runs from ckpt[0] through the h_ref ping-pong
        buffers, the policy (adapters on) through the checkpoints, on the same
        resident copy of the layer.  Same calls on the same inputs as the two
        separate passes, so the same bits, with one layer read fewer."""
        P, N, nl = self.plan, self.n_buffers, self.cfg.n_layers
        for l in range(min(N, nl)):
            self._prefetch(l)
        for l in range(nl):
            base = P.wait(l)
            w = self.views(base)
            h_in = self.ckpt[0] if l == 0 else self.h_ref[(l - 1) % 2]
            L.soup_decoder_layer_fwd(w, self.lora_s[l], self.lcfg, h_in, self.batch, self.seq, self.h_ref[l % 2],
                                     False, self.ws)
            self._policy_fwd(l, w)
            P.release(l)
            if l + N < nl:
                self._prefetch(l + N)

    def _policy_fwd(self, l, w):
        """Layer l's forward pass with the adapters on, keeping what the keep
        plan says for its backward."""
        k = self.keep_plan[l]
        if k == "saved":
            L.soup_decoder_layer_fwd_save(w, self.lora_s[l], self.lcfg, self.ckpt[l], self.batch, self.seq,
                                          self.ckpt[l + 1], True, self.saved[self.saved_row[l]], self.ws)
        elif k == "qkv":
            L.soup_decoder_layer_fwd_keep(w, self.lora_s[l], self.lcfg, self.ckpt[l], self.batch, self.seq,
                                          self.ckpt[l + 1], True, self.keep[self.keep_row[l]], self.ws)
        else:
            L.soup_decoder_layer_fwd(w, self.lora_s[l], self.lcfg, self.ckpt[l], self.batch, self.seq,
                                     self.ckpt[l + 1], True, self.ws)

    def _head(self, coef, logp, dh, h=None):
        P = self.plan
        P.prefetch(self.head_item)
        E = P.wait(self.head_item)
        h = self.ckpt[self.cfg.n_layers] if h is None else h
        if self.prompt_dedup:
            # the rows whose log-probs cover each sequence's continuation (the
            # shared last prompt row read once per sequence of the pair), and
            # their dL/dh summed back onto the token rows in a fixed order
            L.soup_gather_rows(h, self.dd_head_rows, self.h_head)
            L.soup_head_fwd_bwd(self.h_head, self.final_norm, E, self.cfg.vocab, self.cfg.hidden, self.ids_head,
                                self.batch, self.head_seq, self.cfg.eps, self.head_chunk, coef, logp,
                                None if dh is None else self.dh_head, self.head_ws)
            if dh is not None:
                L.soup_sum_rows_f32(self.dh_head, self.dd_src, self.dd_start, dh)
        else:
            L.soup_head_fwd_bwd(h, self.final_norm, E, self.cfg.vocab, self.cfg.hidden,
                                self.ids, self.batch, self.seq, self.cfg.eps, self.head_chunk, coef, logp, dh,
                                self.head_ws)
        P.release(self.head_item)

    def _backward_layers(self):
        P, N, nl = self.plan, self.n_buffers, self.cfg.n_layers
        for l in range(nl - 1, max(nl - 1 - N, -1), -1):
            self._prefetch(l)  # the layers still resident from the forward pass are reused, not copied
        for l in range(nl - 1, -1, -1):
            if self.capture_dh is not None:  # inspection hook for layer-by-layer checks
                self.capture_dh[l + 1] = self.dh.clone()
            base = P.wait(l)
            k = self.keep_plan[l]
            if k == "saved":
                L.soup_decoder_layer_bwd_saved(self.views(base), self.lora_s[l], self.lcfg, self.ckpt[l], self.dh,
                                               self.batch, self.seq, self.dh, self.grads_s[l], 1,
                                               self.saved[self.saved_row[l]], self.ws)
            elif k == "qkv":
                L.soup_decoder_layer_bwd_kept(self.views(base), self.lora_s[l], self.lcfg, self.ckpt[l], self.dh,
                                              self.batch, self.seq, self.dh, self.grads_s[l], 1,
                                              self.keep[self.keep_row[l]], self.ws)
            else:
                L.soup_decoder_layer_bwd(self.views(base), self.lora_s[l], self.lcfg, self.ckpt[l], self.dh,
                                         self.batch, self.seq, self.dh, self.grads_s[l], 1, self.ws)
            P.release(l)
            if l - N >= 0:
                self._prefetch(l - N)
        if self.capture_dh is not None:
            self.capture_dh[0] = self.dh.clone()

    # ------------------------------------------------------------ steps
    def set_ids(self, ids_host):
        """Copies a step's token ids [batch, seq] (pinned int32 host tensor) to the device."""
        self.ids.copy_(ids_host, non_blocking=True)
        if self.prompt_dedup:  # token rows of the shared-prompt layout, and the head's targets
            L.soup_gather_rows(self.ids, self.dd_phys, self.ids_tok)
            L.soup_gather_rows(self.ids, self.dd_head_ids, self.ids_head)

    def sft_step(self):
        """One SFT step on self.ids: next-token CE; leaves LoRA grads in self.grads
        and the loss in self.loss (device)."""
        self._embed()
        self._forward_layers(True)
        L.soup_ce_loss(None, self.batch, self.seq, None, self.coef)
        self._head(self.coef, self.logp, self.dh)
        L.soup_ce_loss(self.logp, self.batch, self.seq, self.loss, None)
        self._backward_layers()
        return self.loss

    def dpo_step(self, prompt_len: int, beta: float):
        """One DPO step on self.ids ([2P, seq]: rows 2p chosen, 2p+1 rejected):
        reference pass with adapters off over the same streamed base, policy
        pass with adapters on, DPO loss, backward through the policy.  A model
        built with task="dpo" runs both forward passes in one visit per layer
        (two layer reads per step instead of three); otherwise they are two
        streamed passes."""
        pairs = self.batch // 2
        self._embed()
        if self.h_ref is not None:
            self._forward_layers_shared()
            self._head(None, self.logp_ref, None, h=self.h_ref[(self.cfg.n_layers - 1) % 2])
        else:
            self._forward_layers(False)
            self._head(None, self.logp_ref, None)
            self._forward_layers(True)
        self._head(None, self.logp, None)
        hs, pl = self._loss_layout(prompt_len)
        L.soup_dpo_loss(self.logp, self.logp_ref, pairs, hs, pl, beta, self.loss, self.seq_sums, self.coef)
        self._head(self.coef, self.logp, self.dh)
        self._backward_layers()
        return self.loss

    def _loss_layout(self, prompt_len):
        """(sequence length, prompt length) of the head's log-probs as the
        preference losses see them: the whole sequences, or with a shared
        prompt stored once only the rows that predict the continuation."""
        if not self.prompt_dedup:
            return self.seq, prompt_len
        if prompt_len != self.prompt_dedup:
            raise ValueError(f"this model shares a {self.prompt_dedup}-token prompt, not {prompt_len}")
        return self.head_seq, 1

    def _preference_step(self, loss_fn):
        """Reference-free preference step: one policy pass (two layer reads
        per step, as for SFT), the loss and dL/dlogp from the sequence sums,
        then the head's backward and the recompute backward."""
        self._embed()
        self._forward_layers(True)
        self._head(None, self.logp, None)
        loss_fn()
        self._head(self.coef, self.logp, self.dh)
        self._backward_layers()
        return self.loss

    def simpo_step(self, prompt_len: int, beta: float = 2.0, gamma: float = 1.0):
        """One SimPO step on self.ids (rows 2p chosen, 2p+1 rejected)."""
        pairs = self.batch // 2
        hs, pl = self._loss_layout(prompt_len)
        return self._preference_step(lambda: L.soup_simpo_loss(self.logp, pairs, hs, pl, beta, gamma,
                                                               self.loss, self.seq_sums, self.coef))

    def orpo_step(self, prompt_len: int, lam: float = 0.1):
        """One ORPO step on self.ids (rows 2p chosen, 2p+1 rejected)."""
        pairs = self.batch // 2
        hs, pl = self._loss_layout(prompt_len)
        return self._preference_step(lambda: L.soup_orpo_loss(self.logp, pairs, hs, pl, lam,
                                                              self.loss, self.seq_sums, self.coef))

    def optimizer_step(self, grad_scale: float = 1.0):
        """AdamW on every LoRA factor: one kernel launch over the flat buffers
        updates the fp32 master copy and the moments, rewrites the bf16 factors
        the next step's GEMMs read, and clears the gradients (the backward pass
        accumulates into them).  grad_scale multiplies the gradients (1/world
        after a data-parallel sum).  A non-finite gradient sets
        self.nonfinite (device) to 1."""
        o = self.adamw
        self.adam_t += 1
        L.soup_adamw_step(self.master_flat, self.lora_flat, self.grad_flat, self.adam_m, self.adam_v, o.lr,
                          o.beta1, o.beta2, o.eps, o.weight_decay, grad_scale, self.adam_t, zero_grad=True,
                          nonfinite=self.nonfinite)

    def forward_logprobs(self, adapters_on=True):
        """Forward only (no grads): per-token log-probs into self.logp."""
        self._embed()
        self._forward_layers(adapters_on)
        self._head(None, self.logp, None)
        return self.logp

    def close(self):
        if getattr(self, "plan", None) is not None:
            self.plan.free()  # synchronises the copy streams first
            self.plan = None
        if getattr(self, "disk", None) is not None:
            self.disk.close()  # staging buffers: no copy reads them any more
            self.disk = None
