"""The output head and the embedding gather at the 8B workload's full size:
vocab 128,256 x hidden 4096 (the lm_head and embed_tokens that share the vocab
slot on the Soup pages, "how layer streaming works"), against the CPU oracle.

* soup_embed gathers the batch's rows straight from the pinned host matrix
  (mapped into the device address space); ids include the last rows of the
  vocabulary, whose byte offsets are the largest.  The gather is bit-exact.
* soup_head_fwd_bwd + soup_ce_loss: final RMSNorm, logits over all 128,256
  rows in token chunks of 256 (the training step's chunk; 258 tokens make a
  full chunk and a ragged one of 2), log-softmax, the CE loss and dL/dh, with
  the split-K dx GEMM over K = 128,256.  logp, dL/dh and the loss within
  relative Frobenius 5e-3 and max|diff| 1e-2 max|ref| of the oracle fed the
  same bf16 inputs.
"""
import numpy as np
import pytest
import torch

import soup_synth as ss
from oracle import head as OH
from tests.gpu_util import assert_close, dev_bf16, host

pytestmark = pytest.mark.gpu

V, H = 128256, 4096


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib as lib
    lib.lib()
    return lib


def _ids(B, S, seed):
    ids = ss.uniform_ids(seed, "fv.ids", (B, S), V)
    # the vocabulary's extreme rows, in several positions (targets and inputs)
    ids[0, :4] = [V - 1, V - 2, 0, V - 1]
    ids[-1, -3:] = [V - 1, 1, V - 2]
    return ids


def test_full_vocab_embed_gather_and_head_match_oracle(L):
    B, S, chunk, eps = 2, 129, 256, 1e-5
    T = B * S
    E = ss.to_bf16_values(ss.normal_f32(21, "fv.lm_head", (V, H), std=0.02))
    wf = ss.to_bf16_values(ss.normal_f32(21, "fv.final_norm", (H,), std=0.02, mean=1.0))
    ids = _ids(B, S, 22)
    ids_d = torch.from_numpy(ids).cuda()

    # embedding gather from pinned host memory: bit-exact rows
    E_host = torch.from_numpy(E).to(torch.bfloat16).pin_memory()
    h_emb = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    L.soup_embed(E_host.data_ptr(), V, H, ids_d, T, h_emb)
    torch.cuda.synchronize()
    assert torch.equal(h_emb.cpu(), E_host[torch.from_numpy(ids.reshape(-1).astype(np.int64))])
    del E_host

    # head: the hidden states are N(0, 1) bf16 (a trained stack's output scale)
    h = ss.to_bf16_values(ss.normal_f32(21, "fv.h", (B, S, H)))
    E_dev = dev_bf16(E)
    hd, wfd = dev_bf16(h.reshape(T, H)), dev_bf16(wf)
    ws = torch.empty(L.soup_head_workspace(V, H, B, S, chunk), dtype=torch.uint8, device="cuda")
    coef = torch.empty((B, S - 1), dtype=torch.float32, device="cuda")
    logp = torch.empty_like(coef)
    dh = torch.empty((T, H), dtype=torch.float32, device="cuda")
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    L.soup_ce_loss(None, B, S, None, coef)
    L.soup_head_fwd_bwd(hd, wfd, E_dev.data_ptr(), V, H, ids_d, B, S, eps, chunk, coef, logp, dh, ws)
    L.soup_ce_loss(logp, B, S, loss, None)
    torch.cuda.synchronize()
    got_logp, got_dh, got_loss = host(logp), host(dh).reshape(B, S, H), float(loss.item())
    del E_dev, ws

    E64 = E.astype(np.float64)
    ref_logp, hc = OH.token_logprobs(h.astype(np.float64), wf, E64, ids, eps, chunk=chunk)
    ref_loss, dlogp = OH.ce_loss(ref_logp)
    ref_dh = OH.token_logprobs_bwd(hc, wf, E64, ids, dlogp, chunk=chunk)
    assert_close(got_logp, ref_logp, "logp (V = 128,256)")
    assert_close(got_dh, ref_dh, "dL/dh (V = 128,256)")
    assert abs(got_loss - ref_loss) <= 5e-3 * abs(ref_loss), (got_loss, ref_loss)
    # an untrained head on random ids: the loss is near ln V
    assert abs(ref_loss - np.log(V)) < 1.0
    assert L.device_error() == 0
