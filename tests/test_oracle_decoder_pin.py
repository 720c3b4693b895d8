"""Pin of the whole oracle decoder against a composition of torch library routines.

The reference below is written from the same page readings (pre/post norms on the
residual, per-head q/k norm before RoPE, scale-free V norm, attention_k_eq_v on
full layers, sliding window attention, GeGLU, layer scalar, tied head, softcap)
but every operation is a torch library call: rms_norm, complex-exponential
rotation for RoPE, scaled_dot_product_attention over the linear history with an
explicit window mask, gelu(approximate="tanh"), tanh. fp16 storage points use
numpy's float16 conversion. Weights come from the oracle's (separately
pinned) q4_0 unpack; the fp16 tied table from the seeded draws rounded by numpy.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import datagen as DG
from datagen import workloads as WL
from oracle import oracle as O


def _h(x: torch.Tensor) -> torch.Tensor:
    # numpy rounds float64 -> float16 directly (nearest even); torch's cast goes
    # through float32 first and double-rounds about 5 values in 10^5.
    return torch.from_numpy(x.numpy().astype(np.float16).astype(np.float64))


def _q8(x: torch.Tensor) -> torch.Tensor:
    """Rows of fp16 values through the int8 KV format, in torch ops: per row a
    float32 scale amax / 127, codes round-half-even(x / scale) clamped to
    [-127, 127] (float32 division), value = code * scale."""
    xf = x.to(torch.float32)
    s = xf.abs().amax(dim=-1, keepdim=True) / torch.tensor(127.0, dtype=torch.float32)
    c = torch.where(s > 0, torch.round(xf / torch.where(s > 0, s, torch.ones_like(s))), torch.zeros_like(xf))
    return c.clamp(-127, 127).to(torch.float64) * s.to(torch.float64)


def _rope(x: torch.Tensor, rot: int, theta: float, pos: int) -> torch.Tensor:
    hd = x.shape[-1]
    half = hd // 2
    i = torch.arange(half, dtype=torch.float64)
    inv = torch.where(i < rot, theta ** (-2.0 * i / hd), torch.zeros_like(i))
    z = torch.complex(x[..., :half], x[..., half:]) * torch.polar(torch.ones_like(inv), pos * inv)
    return torch.cat([z.real, z.imag], dim=-1)


class TorchDecoder:
    def __init__(self, om: O.Model, cfg: dict, seed: int, variant: int):
        self.cfg = cfg
        L = cfg["n_layers"]

        def mat(layer, t):
            got = om.tensor(layer, t)
            return None if got is None else torch.from_numpy(O.q4_0_unpack(*got))

        def gain(stream, n):
            if variant != 1:
                return torch.ones(n, dtype=torch.float64)
            return torch.from_numpy(DG.gain(seed, stream, n).astype(np.float64))

        self.layers = []
        for l in range(L):
            full = WL.layer_is_full(cfg, l)
            hd = cfg["gl_head_dim"] if full else cfg["sl_head_dim"]
            s = lambda t: DG.stream_layer(l, t)
            scal = 1.0 if variant != 1 else float(DG.uniform_float(seed, s(DG.T_LAYER_SCALAR), 1, 0.5, 1.5)[0])
            self.layers.append(dict(
                full=full, hd=hd, wq=mat(l, 0), wk=mat(l, 1), wv=mat(l, 2), wo=mat(l, 3),
                wg=mat(l, 4), wu=mat(l, 5), wd=mat(l, 6),
                n_in=gain(s(DG.T_NORM_IN), cfg["hidden"]), n_pa=gain(s(DG.T_NORM_POST_ATTN), cfg["hidden"]),
                n_pf=gain(s(DG.T_NORM_PRE_FFN), cfg["hidden"]), n_po=gain(s(DG.T_NORM_POST_FFN), cfg["hidden"]),
                n_q=torch.from_numpy(DG.qk_gain(seed, s(DG.T_NORM_Q), hd, variant).astype(np.float64)),
                n_k=torch.from_numpy(DG.qk_gain(seed, s(DG.T_NORM_K), hd, variant).astype(np.float64)),
                scal=scal))
        if cfg.get("head_fp16"):  # the N(0, 0.02) draws rounded to fp16 by numpy
            V, H = cfg["vocab"], cfg["hidden"]
            e = DG.normal(seed, DG.STREAM_EMBED, V * H, 0.02).astype(np.float16)
            self.embed = torch.from_numpy(e.astype(np.float64).reshape(V, H))
        else:
            self.embed = torch.from_numpy(O.q4_0_unpack(*om.tensor(-1, 100)))
        self.n_final = gain(DG.STREAM_FINAL_NORM, cfg["hidden"])
        self.K = [[] for _ in range(L)]   # linear history of fp16 K per layer
        self.V = [[] for _ in range(L)]

    def step(self, token: int, pos: int) -> torch.Tensor:
        c = self.cfg
        eps, H, Hq = c["rms_eps"], c["hidden"], c["n_q_heads"]
        r = self.embed[token] * c["embed_scale"]
        for l, Ly in enumerate(self.layers):
            hd = Ly["hd"]
            nkv = c["gl_kv_heads"] if Ly["full"] else c["sl_kv_heads"]
            rot = c["rope_pairs_full"] if Ly["full"] else hd // 2
            theta = c["rope_theta_gl"] if Ly["full"] else c["rope_theta_sl"]
            x = _h(F.rms_norm(r, (H,), Ly["n_in"], eps))
            q = (Ly["wq"] @ x).view(Hq, hd)
            kraw = (Ly["wk"] @ x).view(nkv, hd)
            vsrc = kraw if Ly["full"] else (Ly["wv"] @ x).view(nkv, hd)
            q = _h(_rope(F.rms_norm(q, (hd,), Ly["n_q"], eps), rot, theta, pos))
            k = _h(_rope(F.rms_norm(kraw, (hd,), Ly["n_k"], eps), rot, theta, pos))
            v = _h(F.rms_norm(vsrc, (hd,), None, eps))
            if c.get("kv_int8"):
                k, v = _q8(k), _q8(v)
            self.K[l].append(k)
            self.V[l].append(v)
            Kh = torch.stack(self.K[l], dim=1)             # [nkv, L, hd]
            Vh = torch.stack(self.V[l], dim=1)
            G = Hq // nkv
            Kh, Vh = Kh.repeat_interleave(G, 0), Vh.repeat_interleave(G, 0)
            mask = torch.ones(Hq, 1, pos + 1, dtype=torch.bool)
            if not Ly["full"]:
                mask[..., : max(0, pos - c["window"] + 1)] = False
            o = F.scaled_dot_product_attention(q[:, None, :], Kh, Vh, attn_mask=mask, scale=1.0)
            o = _h(o.reshape(Hq * hd))
            r = r + F.rms_norm(Ly["wo"] @ o, (H,), Ly["n_pa"], eps)
            x2 = _h(F.rms_norm(r, (H,), Ly["n_pf"], eps))
            a = _h(F.gelu(Ly["wg"] @ x2, approximate="tanh") * (Ly["wu"] @ x2))
            r = (r + F.rms_norm(Ly["wd"] @ a, (H,), Ly["n_po"], eps)) * Ly["scal"]
        z = _h(F.rms_norm(r, (H,), self.n_final, eps))
        return torch.tanh((self.embed @ z) / c["softcap"]) * c["softcap"]


@pytest.mark.parametrize("variant,head_fp16,kv_int8", [(1, 0, 0), (2, 0, 0), (1, 1, 0), (1, 0, 1)])
def test_oracle_decoder_matches_torch_composition(variant, head_fp16, kv_int8):
    """Variant 1: seeded gains and layer scalars; variant 2: unit q/k gains (a sharp
    softmax, logits of order head_dim); head_fp16: the fp16 tied embedding / head;
    kv_int8: K/V rows stored as int8 with a per-row scale."""
    cfg = dict(WL.MICRO, head_fp16=head_fp16, kv_int8=kv_int8)
    seed, steps = 4, 40                      # 40 steps > 2 ring wraps at R = 16
    om = O.Model(cfg, seed=seed, variant=variant)
    cache = O.Cache(om, 64)
    ref = TorchDecoder(om, cfg, seed, variant)
    ids = DG.uniform_int(seed, DG.STREAM_PREFIX_IDS, steps, cfg["vocab"])
    for p in range(steps):
        got = O.decode_step(om, cache, p, token=int(ids[p]))
        want = ref.step(int(ids[p]), p).numpy()
        np.testing.assert_allclose(got["logits"][0], want, rtol=1e-9, atol=1e-10)
        assert got["argmax"][0] == int(np.argmax(want.astype(np.float32)))
