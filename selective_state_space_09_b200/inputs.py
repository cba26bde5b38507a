"""Seeded synthetic inputs for the five scan workloads.

This module only draws random tensors with the shapes and distributions of the workloads; it
holds none of the scan's arithmetic.  Both the CUDA path's tests and the oracle's tests use it,
so that both sides see bit-identical inputs.

Draw order is fixed (the order of the ``_draw`` calls below) and every tensor is drawn in fp32 on
the generator's device and then rounded to the I/O dtype (round-to-nearest-even for bf16).
Parameters (``A``, ``Dskip``, ``mag``, ``theta``) stay fp32.  Key names follow the C ABI's
``lr_inputs`` members (``Bm``, ``Cm``, ``Dskip`` for the selective scans' B, C and D).

Workloads (token-major layouts, last index contiguous):

* ``rglru``  fp32, B=1, D=256, L=1024, segment 128.
  ``a = sigmoid(Lam)^(8 r)``, ``Lam ~ U(2, 6)`` per channel, ``r = sigmoid(N(0,1))`` per step and
  channel; ``b = sqrt(1 - a^2) N(0,1)``.
* ``rglru_gated`` the same shapes with the RG-LRU gate front-end formed in the kernels: inputs
  ``r = sigmoid(N(0,1))``, ``i = sigmoid(N(0,1))``, ``x ~ N(0,1)`` per step and channel and
  ``Lam ~ U(2, 6)`` per channel (key names ``a, b, x, A``: the C ABI members that carry them).
* ``ssd``    bf16 I/O, B=2, H=32, P=64, N=128, L=4096, G=1, ZOH; evaluated in chunks of 128 steps,
  which are also the checkpoint segments.
  ``dt = softplus(N(-2,1))`` per (b,t,h); ``A_h = -exp(U(log 1, log 16))``;
  ``x, B, C ~ N(0,1)/sqrt(N)``; ``D_h ~ N(0,1)``.
* ``gla``    bf16, B=4, H=16, K=V=128, L=2048; chunks (and checkpoint segments) of 128 steps.
  ``g = sigmoid(N(3,1))`` per (b,t,h); ``q, k ~ N(0,1)`` L2-normalised per (b,t,h); ``v ~ N(0,1)``.
* ``s6``     bf16 I/O, B=8, D=2048, N=16, L=2048, segment 64, ZOH or bilinear.
  ``dt = softplus(N(-3,1))``; ``A[d,n] = -(n+1)``; ``B, C ~ N(0,1)`` per (b,t,n); ``x, z, D ~ N(0,1)``.
* ``rotlru`` fp32, B=16, D=4096 (2048 interleaved pairs), L=16384, segment 256.
  ``mag ~ U(0.95, 0.9999)`` and ``theta ~ U(0, pi/8)`` per pair; ``g = sigmoid(N(2,1))`` per
  (b,t,pair); ``b ~ N(0,1)``.

Every workload also draws the upstream gradient ``dy ~ N(0,1)`` with the output's shape.
"""
import math

import torch

WORKLOADS = {
    "rglru": dict(kind="rglru", io="f32", B=1, D=256, L=1024, segment=128),
    "ssd": dict(kind="ssd", io="bf16", B=2, H=32, P=64, N=128, G=1, L=4096, chunk=128,
                segment=128, disc="zoh"),
    "gla": dict(kind="gla", io="bf16", B=4, H=16, K=128, V=128, L=2048, chunk=128, segment=128),
    "s6_zoh": dict(kind="s6", io="bf16", B=8, D=2048, N=16, L=2048, segment=64, disc="zoh"),
    "s6_bilinear": dict(kind="s6", io="bf16", B=8, D=2048, N=16, L=2048, segment=64,
                        disc="bilinear"),
    "rotlru": dict(kind="rotlru", io="f32", B=16, D=4096, L=16384, segment=256),
    # the rglru workload's shapes with the gates formed in the kernels (r, i, x, Lambda)
    "rglru_gated": dict(kind="rglru", io="f32", B=1, D=256, L=1024, segment=128, gates=True),
    # the SSD workload's shapes through the general kernel variant, as Mamba-2 layers run it:
    # dt = softplus(delta + bias) in the kernels, abar = e^{dt A}, beta = dt (ZOH-Euler)
    "ssd_mamba2": dict(kind="ssd", io="bf16", B=2, H=32, P=64, N=128, G=1, L=4096, chunk=128,
                       segment=128, disc="zoh_euler", softplus=True),
    # the SSD workload's inputs through the bilinear (Tustin) discretisation: abar = (1 + u) / (1 - u),
    # u = dt A / 2, negative wherever dt |A| > 2
    "ssd_bilinear": dict(kind="ssd", io="bf16", B=2, H=32, P=64, N=128, G=1, L=4096, chunk=128,
                         segment=128, disc="bilinear"),
}

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


class _Draw:
    def __init__(self, seed, device):
        self.device = torch.device(device)
        self.gen = torch.Generator(device=self.device)
        self.gen.manual_seed(int(seed))

    def randn(self, *shape):
        return torch.randn(*shape, generator=self.gen, device=self.device, dtype=torch.float32)

    def rand(self, *shape):
        return torch.rand(*shape, generator=self.gen, device=self.device, dtype=torch.float32)


def rglru(B, L, D, seed=0, io="f32", device="cpu"):
    r = _Draw(seed, device)
    lam = 2.0 + 4.0 * r.rand(D)
    rr = torch.sigmoid(r.randn(B, L, D))
    a = torch.sigmoid(lam) ** (8.0 * rr)
    b = torch.sqrt(torch.clamp(1.0 - a * a, min=0.0)) * r.randn(B, L, D)
    dy = r.randn(B, L, D)
    t = _DT[io]
    return {"a": a.to(t), "b": b.to(t), "dy": dy.to(t)}


def rglru_gated(B, L, D, seed=0, device="cpu"):
    """Gate-level rglru inputs (f32): a = r (recurrence gate), b = i (input gate), x, A = Lambda."""
    r = _Draw(seed, device)
    lam = 2.0 + 4.0 * r.rand(D)
    rr = torch.sigmoid(r.randn(B, L, D))
    ii = torch.sigmoid(r.randn(B, L, D))
    x = r.randn(B, L, D)
    dy = r.randn(B, L, D)
    return {"a": rr, "b": ii, "x": x, "A": lam, "dy": dy}


def rotlru(B, L, D, seed=0, io="f32", device="cpu"):
    assert D % 2 == 0
    r = _Draw(seed, device)
    K = D // 2
    mag = 0.95 + (0.9999 - 0.95) * r.rand(K)
    theta = (math.pi / 8.0) * r.rand(K)
    g = torch.sigmoid(2.0 + r.randn(B, L, K))
    b = r.randn(B, L, D)
    dy = r.randn(B, L, D)
    t = _DT[io]
    return {"b": b.to(t), "g": g.to(t), "mag": mag, "theta": theta, "dy": dy.to(t)}


def s6(B, L, D, N, seed=0, io="bf16", device="cpu", with_z=True, with_D=True):
    r = _Draw(seed, device)
    x = r.randn(B, L, D)
    delta = torch.nn.functional.softplus(r.randn(B, L, D) - 3.0)
    A = -(torch.arange(N, device=r.device, dtype=torch.float32) + 1.0).repeat(D, 1)
    Bm = r.randn(B, L, N)
    Cm = r.randn(B, L, N)
    Dskip = r.randn(D)
    z = r.randn(B, L, D)
    dy = r.randn(B, L, D)
    t = _DT[io]
    return {"x": x.to(t), "delta": delta.to(t), "A": A.contiguous(), "Bm": Bm.to(t),
            "Cm": Cm.to(t), "Dskip": Dskip if with_D else None, "z": z.to(t) if with_z else None,
            "dy": dy.to(t)}


def ssd(B, L, H, P, N, G=1, seed=0, io="bf16", device="cpu", with_z=False, with_D=True):
    assert H % G == 0
    r = _Draw(seed, device)
    s = 1.0 / math.sqrt(N)
    x = r.randn(B, L, H, P) * s
    delta = torch.nn.functional.softplus(r.randn(B, L, H) - 2.0)
    A = -torch.exp(math.log(16.0) * r.rand(H))
    Bm = r.randn(B, L, G, N) * s
    Cm = r.randn(B, L, G, N) * s
    Dskip = r.randn(H)
    dy = r.randn(B, L, H, P)
    z = r.randn(B, L, H, P) if with_z else None
    t = _DT[io]
    return {"x": x.to(t), "delta": delta.to(t), "A": A, "Bm": Bm.to(t), "Cm": Cm.to(t),
            "Dskip": Dskip if with_D else None, "z": z.to(t) if z is not None else None,
            "dy": dy.to(t)}


def gla(B, L, H, K, V, seed=0, io="bf16", device="cpu"):
    r = _Draw(seed, device)
    g = torch.sigmoid(3.0 + r.randn(B, L, H))
    q = r.randn(B, L, H, K)
    k = r.randn(B, L, H, K)
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    v = r.randn(B, L, H, V)
    dy = r.randn(B, L, H, V)
    t = _DT[io]
    return {"q": q.to(t), "k": k.to(t), "v": v.to(t), "g": g.to(t), "dy": dy.to(t)}


def workload(name, seed=0, device="cpu", **override):
    """Inputs for one named workload; ``override`` replaces shape keys (B, L, ...)."""
    w = dict(WORKLOADS[name])
    w.update(override)
    k = w["kind"]
    if k == "rglru" and w.get("gates"):
        return rglru_gated(w["B"], w["L"], w["D"], seed, device)
    if k == "rglru":
        return rglru(w["B"], w["L"], w["D"], seed, w["io"], device)
    if k == "rotlru":
        return rotlru(w["B"], w["L"], w["D"], seed, w["io"], device)
    if k == "s6":
        return s6(w["B"], w["L"], w["D"], w["N"], seed, w["io"], device)
    if k == "ssd":
        inp = ssd(w["B"], w["L"], w["H"], w["P"], w["N"], w.get("G", 1), seed, w["io"], device)
        if w.get("softplus"):  # raw step lengths N(-2, 1) and a bias U(-1, 0) per head, drawn after
            g = torch.Generator(device="cpu").manual_seed(seed + 7919)
            raw = torch.randn(inp["delta"].shape, generator=g) - 2.0
            inp["delta"] = raw.to(_DT[w["io"]]).to(device)
            inp["delta_bias"] = (-torch.rand(w["H"], generator=g)).to(device)
        return inp
    if k == "gla":
        return gla(w["B"], w["L"], w["H"], w["K"], w["V"], seed, w["io"], device)
    raise KeyError(k)
