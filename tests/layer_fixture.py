"""Builds one decoder layer's frozen base and LoRA factors on the GPU from the
seeded synthetic inputs (soup_synth), together with the oracle's view of the
same layer (dequantised weights as fp64).  Used by the GPU layer tests."""
import numpy as np
import torch

import soup_synth as ss
from oracle import nf4 as onf4
from tests.gpu_util import dev_bf16, dev_f32


def quantize_dev(L, W32):
    out_f, in_f = W32.shape
    codes = torch.empty((out_f, in_f // 2), dtype=torch.uint8, device="cuda")
    absmax = torch.empty((out_f, in_f // 64), dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.soup_nf4_quantize(dev_f32(W32), codes, absmax, flag)
    return codes, absmax


class DevLayer:
    """Device tensors of one layer + the ctypes structs pointing at them."""

    def __init__(self, L, shape, seed=0, layer=0, kind="nf4", zero_B=False, lora_std=0.02, check_codes=False):
        self.shape = shape
        Wf = ss.layer_weights_f32(shape, seed, layer)
        lo = ss.lora_params(shape, seed, layer, std=lora_std, zero_B=zero_B)
        fused = {
            "qkv": np.concatenate([Wf["q"], Wf["k"], Wf["v"]]),
            "o": Wf["o"],
            "gate_up": np.concatenate([Wf["gate"], Wf["up"]]),
            "down": Wf["down"],
        }
        self.keep = []
        structs = {}
        self.W_oracle = {}
        for name, W32 in fused.items():
            if kind == "nf4":
                # the GPU quantises the fp32 weights; the oracle quantises the
                # same weights itself (no oracle input comes from the GPU)
                codes, absmax = quantize_dev(L, W32)
                self.keep += [codes, absmax]
                structs[name] = L.weight_nf4(codes, absmax, *W32.shape)
                packed, am = onf4.quantize(W32)
                if check_codes:
                    assert np.array_equal(codes.cpu().numpy(), packed), f"{name}: NF4 codes differ"
                    assert np.array_equal(absmax.cpu().numpy(), am), f"{name}: absmax differs"
                deq = onf4.dequant_bf16(packed, am).astype(np.float64)
                del packed, am
            elif kind == "nf4_stored":
                # stored NF4 weights drawn directly (full-size layers: the
                # oracle only dequantises, no fp64 quantisation of 218 M weights)
                packed, am = ss.nf4_stored_blocks(seed, f"{layer}.{name}.nf4", *W32.shape)
                codes = torch.from_numpy(packed).cuda()
                absmax = torch.from_numpy(am).cuda()
                self.keep += [codes, absmax]
                structs[name] = L.weight_nf4(codes, absmax, *W32.shape)
                deq = onf4.dequant_bf16(packed, am).astype(np.float64)
            else:
                deq = onf4.round_to_bf16(W32).astype(np.float64)
                wb = dev_bf16(deq)
                self.keep.append(wb)
                structs[name] = L.weight_bf16(wb)
            self.W_oracle[name] = deq
        qo, ko = shape.n_q_heads * shape.head_dim, shape.n_kv_heads * shape.head_dim
        I = shape.intermediate
        d = self.W_oracle
        self.Wd = {"q": d["qkv"][:qo], "k": d["qkv"][qo:qo + ko], "v": d["qkv"][qo + ko:],
                   "o": d["o"], "gate": d["gate_up"][:I], "up": d["gate_up"][I:], "down": d["down"],
                   "norm1": Wf["norm1"].astype(np.float64), "norm2": Wf["norm2"].astype(np.float64)}
        self.norm1, self.norm2 = dev_bf16(Wf["norm1"]), dev_bf16(Wf["norm2"])
        self.W = L.LayerWeights(structs["qkv"], structs["o"], structs["gate_up"], structs["down"],
                                self.norm1.data_ptr(), self.norm2.data_ptr())
        self.lora_np = {p: (lo[p][0].astype(np.float64), lo[p][1].astype(np.float64)) for p in ss.PROJ_NAMES}
        cat = lambda ps, i: np.concatenate([lo[p][i] for p in ps])
        self.lora_t = {
            "A_qkv": dev_bf16(cat(("q", "k", "v"), 0)), "B_qkv": dev_bf16(cat(("q", "k", "v"), 1)),
            "A_o": dev_bf16(lo["o"][0]), "B_o": dev_bf16(lo["o"][1]),
            "A_gu": dev_bf16(cat(("gate", "up"), 0)), "B_gu": dev_bf16(cat(("gate", "up"), 1)),
            "A_down": dev_bf16(lo["down"][0]), "B_down": dev_bf16(lo["down"][1]),
        }
        self.lora = L.layer_lora(self.lora_t)
        self.grads_t = {"d" + k: torch.zeros(v.shape, dtype=torch.float32, device="cuda")
                        for k, v in self.lora_t.items()}
        self.grads = L.layer_grads(self.grads_t)
        self.cfg = L.layer_cfg(shape)

    def split_grads(self):
        """GPU grads -> dict proj -> (dA, dB) numpy, in the oracle's layout."""
        g = {k: v.cpu().numpy().astype(np.float64) for k, v in self.grads_t.items()}
        s = self.shape
        r, qo, ko, I = s.rank, s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim, s.intermediate
        return {
            "q": (g["dA_qkv"][:r], g["dB_qkv"][:qo]),
            "k": (g["dA_qkv"][r:2 * r], g["dB_qkv"][qo:qo + ko]),
            "v": (g["dA_qkv"][2 * r:], g["dB_qkv"][qo + ko:]),
            "o": (g["dA_o"], g["dB_o"]),
            "gate": (g["dA_gu"][:r], g["dB_gu"][:I]),
            "up": (g["dA_gu"][r:], g["dB_gu"][I:]),
            "down": (g["dA_down"], g["dB_down"]),
        }
