"""Seeded synthetic weights for the streamed model built from soup_synth on the
host, so that the CPU oracle can be given exactly the same values."""
import numpy as np
import torch

import soup_synth as ss
from oracle import nf4 as onf4


def shape_of(cfg):
    return ss.LayerShape(hidden=cfg.hidden, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                         intermediate=cfg.intermediate, rank=cfg.rank, alpha=cfg.alpha, eps=cfg.eps, theta=cfg.theta,
                         vocab=cfg.vocab, n_layers=cfg.n_layers)


class NumpyWeights:
    def __init__(self, cfg, seed=0):
        self.cfg = cfg
        self.shape = shape_of(cfg)
        self.seed = seed
        self.f32 = [ss.layer_weights_f32(self.shape, seed, l) for l in range(cfg.n_layers)]
        self.lo = [ss.lora_params(self.shape, seed, l) for l in range(cfg.n_layers)]
        V, H = cfg.vocab, cfg.hidden
        self.embed = ss.to_bf16_values(ss.normal_f32(seed, "embed", (V, H), std=0.02))
        self.head = self.embed if cfg.tied else ss.to_bf16_values(ss.normal_f32(seed, "lm_head", (V, H), std=0.02))
        self.final = ss.to_bf16_values(ss.normal_f32(seed, "final_norm", (H,), std=0.02, mean=1.0))

    # ---- device side (the model under test)
    def layer(self, l):
        w = self.f32[l]
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
        return {"qkv": dev(np.concatenate([w["q"], w["k"], w["v"]])), "o": dev(w["o"]),
                "gate_up": dev(np.concatenate([w["gate"], w["up"]])), "down": dev(w["down"]),
                "norm1": dev(w["norm1"]).to(torch.bfloat16), "norm2": dev(w["norm2"]).to(torch.bfloat16)}

    def vocab(self, which):
        a = self.embed if which == "embed" else self.head
        return torch.from_numpy(a).cuda().to(torch.bfloat16)

    def final_norm(self):
        return torch.from_numpy(self.final).cuda().to(torch.bfloat16)

    def lora(self, l):
        lo = self.lo[l]
        cat = lambda ps, i: np.concatenate([lo[p][i] for p in ps])
        arrs = {"A_qkv": cat(("q", "k", "v"), 0), "B_qkv": cat(("q", "k", "v"), 1), "A_o": lo["o"][0],
                "B_o": lo["o"][1], "A_gu": cat(("gate", "up"), 0), "B_gu": cat(("gate", "up"), 1),
                "A_down": lo["down"][0], "B_down": lo["down"][1]}
        return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda().to(torch.bfloat16) for k, v in arrs.items()}

    # ---- oracle side
    def oracle_params(self):
        layers = []
        for l in range(self.cfg.n_layers):
            w = self.f32[l]
            if self.cfg.kind == "nf4":
                Wd = {p: onf4.dequant_bf16(*onf4.quantize(w[p])).astype(np.float64) for p in ss.PROJ_NAMES}
            else:
                Wd = {p: onf4.round_to_bf16(w[p]).astype(np.float64) for p in ss.PROJ_NAMES}
            Wd["norm1"] = w["norm1"].astype(np.float64)
            Wd["norm2"] = w["norm2"].astype(np.float64)
            lora = {p: (self.lo[l][p][0].astype(np.float64), self.lo[l][p][1].astype(np.float64))
                    for p in ss.PROJ_NAMES}
            layers.append((Wd, lora))
        return dict(layers=layers, embed=self.embed.astype(np.float64), head=self.head.astype(np.float64),
                    final_norm=self.final.astype(np.float64))


def split_grads(cfg, g):
    """Fused GPU grads (dict of torch fp32) -> proj -> (dA, dB) numpy."""
    g = {k: v.cpu().numpy().astype(np.float64) for k, v in g.items()}
    r, qo, ko, I = cfg.rank, cfg.n_q_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.intermediate
    return {
        "q": (g["dA_qkv"][:r], g["dB_qkv"][:qo]), "k": (g["dA_qkv"][r:2 * r], g["dB_qkv"][qo:qo + ko]),
        "v": (g["dA_qkv"][2 * r:], g["dB_qkv"][qo + ko:]), "o": (g["dA_o"], g["dB_o"]),
        "gate": (g["dA_gu"][:r], g["dB_gu"][:I]), "up": (g["dA_gu"][r:], g["dB_gu"][I:]),
        "down": (g["dA_down"], g["dB_down"]),
    }
