"""Seeded synthetic workloads for the LSA layer.

This module holds random-number recipes only -- none of the method's arithmetic (no scores,
no selection, no attention).  The tests, the benchmark and the smoke check draw their inputs
here, and both the CUDA path and the CPU oracle read the same bytes.

bf16 tensors are produced by rounding float32 draws to nearest-even once; on the host they are
``uint16`` bit patterns, on the device ``torch.bfloat16``.

Recipes (shapes and distributions of the paper's workloads, LongCat Sparse Attention,
Sec. 2.3 Table 1, Sec. 4.1 Tables 3-4, Sec. 5.1 Table 6):
  * indexer q, k ~ N(0,1)/sqrt(d_I); head weights w ~ U(0,1) (tiny case) or softplus(N(0,1));
  * MLA latent rows c (576 = 512 + 64 dims) and MLA queries ~ N(0,1);
  * planted "needles": a key made to align with a late query's head-weighted indexer query
    (3x a typical key norm), and its latent row aligned with that query's mean MLA query;
  * clustered topics for prefill: 32 centres, contiguous topic spans of geometric length
    (mean 512), per-token noise sigma = 0.5.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

D_QK = 576  # MLA latent row: 512 (kv LoRA rank) + 64 (rope)
D_V = 512


# ----------------------------------------------------------------------------- bf16 bits

def to_bf16_bits(x) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def softplus(x):
    return np.log1p(np.exp(-np.abs(x))) + np.maximum(x, 0)


# ----------------------------------------------------------------------------- configs

@dataclass(frozen=True)
class LsaConfig:
    name: str
    B: int                 # sequences
    L: int                 # cached tokens per sequence (kv_len)
    T: int                 # queries per sequence in one call
    H_I: int = 64          # indexer heads
    D_I: int = 128         # indexer head dim
    H: int = 128           # MLA heads
    K: int = 2048          # total budget = sink + swa + sparse
    sink: int = 16
    swa: int = 1024
    page: int = 128
    sub_block: int = 8
    M: int = 0             # recalled pages (0 = flat indexer)
    w_dist: str = "softplus"
    topics: bool = False
    n_needles: int = 64
    needle_pages: int = 0  # >0: needles confined to this many random pages
    chunk: int = 0         # prefill query chunk (0 = all T at once)
    layers: int = 2        # CLI group size N (owner + reuse layers)
    seed: int = 0
    L_max: int = 0         # cache capacity (0 = L)
    scale: float = 1.0 / 24.0  # 1/sqrt(576)

    @property
    def K_sparse(self) -> int:
        return self.K - self.sink - self.swa

    @property
    def cap(self) -> int:
        return self.L_max if self.L_max else self.L


TINY = LsaConfig("tiny_prefill_1k", B=1, L=1024, T=1024, H_I=8, D_I=64, H=8, K=256, sink=16,
                 swa=128, w_dist="uniform", n_needles=8, layers=1)
DECODE_128K = LsaConfig("decode_b32_128k_cli2", B=32, L=131072, T=1)
PREFILL_32K = LsaConfig("prefill_b1_32k_chunk4096", B=1, L=32768, T=32768, topics=True,
                        n_needles=0, chunk=4096, layers=1)
DECODE_1M_HI = LsaConfig("decode_b4_1m_hi", B=4, L=1048576, T=1, M=1024, needle_pages=256)
SWEEP_LENGTHS = (4096, 16384, 65536, 131072, 262144, 524288, 1048576)


def sweep_config(L: int, variant: str) -> LsaConfig:
    """Table-1-shaped decode sweep point: 'dsa' = flat 2048 dynamic top-K, no sink/swa;
    'lsa' = SI + HI from 256K + CLI N=2."""
    if variant not in ("dsa", "lsa"):
        raise ValueError(f"sweep variant {variant!r}: 'dsa' or 'lsa'")
    base = LsaConfig(f"sweep_b8_{L}_{variant}", B=8, L=L, T=1)
    if variant == "dsa":
        # one indexer pass per layer (no cross-layer reuse)
        return replace(base, sink=0, swa=0, K=2048, M=0, layers=1)
    return replace(base, M=1024 if L >= 262144 else 0)


INDEX_CHUNK_LENGTHS = (32768, 65536, 131072, 262144, 524288, 1048576)


def index_chunk_config(L: int, variant: str) -> LsaConfig:
    """Indexer of one prefill chunk (the paper's Table 4 setting): the last 2048 queries of a
    single L-token sequence, hierarchical ('hi': P=128, 8-token sub-blocks, M=1024 pages) or flat
    ('flat')."""
    if variant not in ("hi", "flat"):
        raise ValueError(f"index chunk variant {variant!r}: 'hi' or 'flat'")
    return LsaConfig(f"index_chunk_2048q_{L}_{variant}", B=1, L=L, T=2048,
                     M=1024 if variant == "hi" else 0, needle_pages=256, layers=1)


TRAIN_LENGTHS = (8192, 16384, 32768, 65536, 131072, 262144, 524288, 1048576)


def train_config(L: int) -> LsaConfig:
    """Core attention of one training step (the paper's Table 2 setting): batch 1, the last 8192
    queries of an L-token sequence, 128 heads, K = 2048 = 16 sink + 1024 window + 1008 dynamic."""
    if L < 8192:
        raise ValueError("the training workload needs L >= 8192 (8192 queries)")
    return LsaConfig(f"hfa_train_b1_q8192_{L}", B=1, L=L, T=8192, layers=1)


CONFIGS = {c.name: c for c in (TINY, DECODE_128K, PREFILL_32K, DECODE_1M_HI)}


# ----------------------------------------------------------------------------- host (numpy)

@dataclass
class HostInputs:
    cfg: LsaConfig
    q_I: np.ndarray          # [B,T,H_I,D_I] bf16 bits
    w_I: np.ndarray          # [B,T,H_I]
    k_I: np.ndarray          # [B,cap,D_I]
    q: list = field(default_factory=list)      # per layer [B,T,H,576]
    c_kv: list = field(default_factory=list)   # per layer [B,cap,576]
    kv_len: np.ndarray = None  # [B] int32
    q_pos: np.ndarray = None   # [B,T] int32
    needles: np.ndarray = None  # [B, n] int64 planted positions (-1 none)


def _rows_normalise(x):
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    return x / np.maximum(n, 1e-30)


def make_host_inputs(cfg: LsaConfig, seed: int | None = None, q_pos=None, kv_len=None,
                     with_attention: bool = True) -> HostInputs:
    """Numpy recipe for sizes the oracle can digest (tests, smoke).  q_pos default: the last T
    positions of each sequence (decode when T == 1, all queries when T == L)."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    B, L, T, HI, DI, H, cap = cfg.B, cfg.L, cfg.T, cfg.H_I, cfg.D_I, cfg.H, cfg.cap
    if kv_len is None:
        kv_len = np.full(B, L, dtype=np.int32)
    kv_len = np.asarray(kv_len, dtype=np.int32)
    if q_pos is None:
        q_pos = np.stack([np.arange(kv_len[b] - T, kv_len[b]) for b in range(B)]).astype(np.int32)
    q_pos = np.asarray(q_pos, dtype=np.int32).reshape(B, T)

    sig = 1.0 / np.sqrt(DI)
    if cfg.topics:
        centres = rng.standard_normal((32, DI)).astype(np.float32)
        topic = _topic_track(rng, cap)
        k = (centres[topic] + 0.5 * rng.standard_normal((B, cap, DI))) * sig
        qt = topic[np.clip(q_pos, 0, cap - 1)]                       # [B,T]
        qI = (centres[qt][:, :, None, :] + 0.5 * rng.standard_normal((B, T, HI, DI))) * sig
    else:
        k = rng.standard_normal((B, cap, DI)) * sig
        qI = rng.standard_normal((B, T, HI, DI)) * sig
    if cfg.w_dist == "uniform":
        w = rng.random((B, T, HI))
    else:
        w = softplus(rng.standard_normal((B, T, HI)))
    qI = qI.astype(np.float32)
    w = w.astype(np.float32)
    k = k.astype(np.float32)

    qm, cm = [], []
    if with_attention:
        for _layer in range(cfg.layers):
            if cfg.topics:
                cc = rng.standard_normal((32, D_QK)).astype(np.float32)
                c = cc[topic] + 0.5 * rng.standard_normal((B, cap, D_QK))
                qq = rng.standard_normal((B, T, H, D_QK)) + cc[qt][:, :, None, :]
            else:
                c = rng.standard_normal((B, cap, D_QK))
                qq = rng.standard_normal((B, T, H, D_QK))
            qm.append(qq.astype(np.float32))
            cm.append(c.astype(np.float32))

    needles = _plant_needles_host(rng, cfg, qI, w, k, qm, cm, q_pos)
    return HostInputs(cfg=cfg, q_I=to_bf16_bits(qI), w_I=to_bf16_bits(w), k_I=to_bf16_bits(k),
                      q=[to_bf16_bits(x) for x in qm], c_kv=[to_bf16_bits(x) for x in cm],
                      kv_len=kv_len, q_pos=q_pos, needles=needles)


def _topic_track(rng, n):
    """Topic id per position: contiguous spans with geometric lengths (mean 512)."""
    out = np.empty(n, dtype=np.int64)
    s = 0
    while s < n:
        ln = int(rng.geometric(1.0 / 512.0))
        out[s:s + ln] = rng.integers(0, 32)
        s += ln
    return out


def _plant_needles_host(rng, cfg, qI, w, k, qm, cm, q_pos):
    B, T = q_pos.shape
    n = cfg.n_needles
    needles = np.full((B, max(n, 1)), -1, dtype=np.int64)
    if n == 0:
        return needles
    knorm = np.sqrt(cfg.D_I) / np.sqrt(cfg.D_I)  # typical |k| for N(0, 1/D) rows = 1
    cnorm = np.sqrt(D_QK)
    for b in range(B):
        late = np.arange(T)[q_pos[b] >= 0]
        late = late[-max(1, T // 8):]          # late queries of this sequence
        for i in range(n):
            ti = int(rng.choice(late))
            t = int(q_pos[b, ti])
            lo, hi = cfg.sink, t - cfg.swa + 1
            if hi <= lo:
                continue
            p = int(rng.integers(lo, hi))
            needles[b, i] = p
            dirk = (w[b, ti][:, None] * qI[b, ti]).sum(0)
            k[b, p] = 3.0 * knorm * _rows_normalise(dirk)
            for layer in range(len(cm)):
                dirc = qm[layer][b, ti].mean(0)
                cm[layer][b, p] = 3.0 * cnorm * _rows_normalise(dirc)
    return needles


# ----------------------------------------------------------------------------- device (torch)

class DeviceInputs:
    """Large workloads drawn directly on the GPU with torch's seeded Philox generator (the
    oracle then reads back the rows it samples).  Tensors: q_I [B,T,H_I,D_I], w_I [B,T,H_I],
    k_I [B,cap,D_I], k_mean [B,ceil(cap/sub),D_I] (zeros; filled by the append kernel), per layer
    q [B,T,H,576] and c_kv [B,cap,576], kv_len [B] int32, q_pos [B,T] int32."""

    def __init__(self, cfg: LsaConfig, device="cuda", seed: int | None = None,
                 with_attention: bool = True):
        import torch
        self.cfg = cfg
        g = torch.Generator(device=device)
        g.manual_seed(cfg.seed if seed is None else seed)
        B, L, T, HI, DI, H, cap = cfg.B, cfg.L, cfg.T, cfg.H_I, cfg.D_I, cfg.H, cfg.cap
        bf = torch.bfloat16
        sig = 1.0 / float(np.sqrt(DI))

        def randn(*shape, scale=1.0, dtype=bf):
            # generate in bounded slabs so peak fp32 scratch stays small
            out = torch.empty(*shape, dtype=dtype, device=device)
            flat = out.view(-1)
            step = 1 << 26
            for s in range(0, flat.numel(), step):
                e = min(flat.numel(), s + step)
                flat[s:e] = (torch.randn(e - s, generator=g, device=device) * scale).to(dtype)
            return out

        self.kv_len = torch.full((B,), L, dtype=torch.int32, device=device)
        self.q_pos = (torch.arange(L - T, L, dtype=torch.int32, device=device)
                      .unsqueeze(0).repeat(B, 1).contiguous())
        if cfg.topics:
            centres = torch.randn(32, DI, generator=g, device=device)
            topic = torch.as_tensor(_topic_track(np.random.default_rng(cfg.seed + 7), cap),
                                    device=device)
            self.k_I = ((centres[topic].unsqueeze(0)
                         + 0.5 * torch.randn(B, cap, DI, generator=g, device=device)) * sig).to(bf)
            qt = topic[self.q_pos.long().clamp(0, cap - 1)]
            self.q_I = ((centres[qt].unsqueeze(2)
                         + 0.5 * torch.randn(B, T, HI, DI, generator=g, device=device))
                        * sig).to(bf)
        else:
            self.k_I = randn(B, cap, DI, scale=sig)
            self.q_I = randn(B, T, HI, DI, scale=sig)
        if cfg.w_dist == "uniform":
            self.w_I = torch.rand(B, T, HI, generator=g, device=device).to(bf)
        else:
            self.w_I = torch.nn.functional.softplus(
                torch.randn(B, T, HI, generator=g, device=device)).to(bf)
        nb = (cap + cfg.sub_block - 1) // cfg.sub_block
        self.k_mean = torch.zeros(B, nb, DI, dtype=bf, device=device)
        self.q, self.c_kv = [], []
        if with_attention:
            for _layer in range(cfg.layers):
                if cfg.topics:
                    cc = torch.randn(32, D_QK, generator=g, device=device)
                    c = (cc[topic].unsqueeze(0)
                         + 0.5 * torch.randn(B, cap, D_QK, generator=g, device=device)).to(bf)
                    qq = (torch.randn(B, T, H, D_QK, generator=g, device=device)
                          + cc[qt].unsqueeze(2)).to(bf)
                else:
                    c = randn(B, cap, D_QK)
                    qq = randn(B, T, H, D_QK)
                self.c_kv.append(c)
                self.q.append(qq)
        self.needles = self._plant(g)

    def _plant(self, g):
        import torch
        cfg = self.cfg
        B, T = cfg.B, cfg.T
        n = cfg.n_needles
        if n == 0:
            return None
        rng = np.random.default_rng(cfg.seed + 11)
        pos = np.full((B, n), -1, dtype=np.int64)
        q_pos = self.q_pos.cpu().numpy()
        for b in range(B):
            for i in range(n):
                ti = int(rng.integers(max(0, T - max(1, T // 8)), T))
                t = int(q_pos[b, ti])
                lo, hi = cfg.sink, t - cfg.swa + 1
                if hi <= lo:
                    continue
                if cfg.needle_pages:
                    pages = rng.choice(np.arange(lo // cfg.page, (hi - 1) // cfg.page + 1),
                                       size=1)
                    p = int(np.clip(pages[0] * cfg.page + rng.integers(0, cfg.page), lo, hi - 1))
                else:
                    p = int(rng.integers(lo, hi))
                pos[b, i] = p
                wq = (self.w_I[b, ti].float()[:, None] * self.q_I[b, ti].float()).sum(0)
                self.k_I[b, p] = (3.0 * wq / wq.norm().clamp_min(1e-30)).to(self.k_I.dtype)
                for layer in range(len(self.c_kv)):
                    dq = self.q[layer][b, ti].float().mean(0)
                    self.c_kv[layer][b, p] = (3.0 * float(np.sqrt(D_QK)) * dq
                                              / dq.norm().clamp_min(1e-30)).to(torch.bfloat16)
        return pos
