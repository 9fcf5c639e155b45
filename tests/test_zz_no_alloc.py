"""lsa_index_noalloc: the indexer entry point for callers that cannot allocate device memory
(for example a plug-in inside an application whose memory pool owns the whole GPU, or a serving
loop that forbids cudaMalloc on its hot path).  It must give exactly the indices that lsa_index
gives with a caller-provided workspace, on consecutive calls that share the library's fixed
scratch array.  This file is collected last on purpose."""
import numpy as np
import pytest

from lightning_indexer_top_score_b200 import lsa
from lightning_indexer_top_score_b200.workloads import LsaConfig, make_host_inputs
from _tensors import dev_bf16, dev_i32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _inputs(seed, M):
    cfg = LsaConfig("noalloc", B=4, L=20000, T=2, K=16 + 1024 + 1008, sink=16, swa=1024,
                    n_needles=8, seed=seed, M=M)
    h = make_host_inputs(cfg, q_pos=np.array([[19999, 15000]] * 4, np.int32), with_attention=False)
    q, w, k = dev_bf16(h.q_I), dev_bf16(h.w_I), dev_bf16(h.k_I)
    km = None
    if M:
        nb = (cfg.L + cfg.sub_block - 1) // cfg.sub_block
        km = torch.zeros(cfg.B, nb, cfg.D_I, dtype=torch.bfloat16, device="cuda")
        lsa.lsa_kv_append(dev_i32(np.zeros(cfg.B, np.int32)), k_I_new=k.clone(), k_I=k,
                          k_mean=km, sub_block=cfg.sub_block)
    return cfg, q, w, k, km, dev_i32(h.kv_len), dev_i32(h.q_pos)


@pytest.mark.parametrize("M", [0, 16])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(M):
    for seed in (21, 22):  # two calls in a row share (and must re-clear) the static scratch
        cfg, q, w, k, km, kv, qp = _inputs(seed, M)
        ref = lsa.lsa_index(q, w, k, km, kv, qp, cfg.K_sparse, cfg.sink, cfg.swa, cfg.page,
                            cfg.sub_block, M)
        err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        got = lsa.lsa_index_noalloc(q, w, k, km, kv, qp, cfg.K_sparse, cfg.sink, cfg.swa,
                                    cfg.page, cfg.sub_block, M, device_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(got, ref), f"seed {seed}"
        assert int((got[:, 0] >= 0).sum(-1).min().item()) == cfg.K_sparse


def test_noalloc_rejects_sizes_beyond_its_scratch():
    need = lsa.lsa_index_workspace_bytes(64, 1, 64, 128, 1 << 20, 1008)
    assert need > lsa.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = lsa.load().lsa_index_noalloc(
        lsa._ptr(x), lsa._ptr(x), lsa._ptr(x), None, lsa._ptr(i), lsa._ptr(i), 64, 1, 64, 128,
        1 << 20, 1008, 16, 1024, 128, 8, 0, lsa._ptr(i), None, lsa._stream(None))
    assert st == 3  # LSA_ERR_WORKSPACE, before any device work
