"""Runs the hot path on small ragged shapes through libheal_debug.so (the kernels built
with HEAL_DEBUG: every global store index they compute is checked in the kernel, and a
violation is reported by heal_get_device_status() instead of faulting).

Run as a separate process (the library choice is per process) by
tests/test_gpu_debug_build.py; prints one JSON object: for each case whether the device
status stayed clean and whether the result matches the oracle.
"""
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import error_compensated_gemm_b200._binding as B  # noqa: E402

B.use_debug_library()
import synthetic  # noqa: E402
from oracle import attention as OA  # noqa: E402
from oracle import gemm as OG  # noqa: E402
from oracle import quant as OQ  # noqa: E402
from oracle import split as OS  # noqa: E402

d = torch.device("cuda:0")
res = {}


def status():
    torch.cuda.synchronize()
    return B.heal_get_device_status()


def gemm_case(M, N, K, tile, b_layout=0, presplit=False):
    X, W = synthetic.gemm_prefill(M=M, K=K, N=N)
    Bin = W if b_layout == 0 else W.t().contiguous()
    Xd, Bd = X.to(d), Bin.to(d).contiguous()
    C = torch.full((M, N), float("nan"), device=d)
    nb = B.heal_gemm_workspace_bytes(M, N, K, tile)
    ws = torch.empty(max(nb, 16) // 4, device=d) if nb else None
    if presplit:
        hi = torch.empty(Bd.shape, dtype=torch.int16, device=d)
        lo = torch.empty_like(hi)
        B.heal_split(Bd, hi, lo)
        B.heal_gemm_compensated(Xd, hi, C, tile_config=tile, b_layout=b_layout, b_lo=lo, workspace=ws)
    else:
        B.heal_gemm_compensated(Xd, Bd, C, tile_config=tile, b_layout=b_layout, workspace=ws)
    st = status()
    c = C.cpu().numpy().astype(np.float64)
    err = OG.normwise_rel_err(c, OG.gemm_ref(X.numpy(), W.numpy()))
    return {"status": st, "err": err, "ok": st == B.HEAL_OK and err <= 1e-6}, c


gemm_bits = {}
# ragged against the 128/256 tiles and the 64-wide chunks; row strides stay multiples of 8
for (M, N, K) in ((200, 296, 328), (5, 648, 136), (33, 1000, 1000), (300, 520, 200)):
    for tile in (B.TILE_128x128, B.TILE_256x256_PAIR, B.TILE_SKINNY_SPLITK, B.TILE_SKINNY_FULLK,
                 B.TILE_SKINNY_CHAIN):
        if tile in (B.TILE_SKINNY_SPLITK, B.TILE_SKINNY_FULLK, B.TILE_SKINNY_CHAIN) and M > 64:
            continue
        for b_layout in (0, 1):
            r, c = gemm_case(M, N, K, tile, b_layout)
            res[f"gemm_{M}x{N}x{K}_tile{tile}_layout{b_layout}"] = r
            gemm_bits.setdefault((M, N, K), []).append(c)
    r, c = gemm_case(M, N, K, B.TILE_AUTO, 0, presplit=True)
    res[f"gemm_{M}x{N}x{K}_presplit"] = r
    gemm_bits[(M, N, K)].append(c)
res["gemm_bits_identical_across_configs"] = {
    "ok": all(all(np.array_equal(c, v[0]) for c in v[1:]) for v in gemm_bits.values())}

# split: ragged length (vector body and scalar tail), bit-exact encodings
x = synthetic.with_outliers(synthetic.normal((1, 10001), seed=3), 0.05, 20.0, seed=4).numpy().ravel()
xd = torch.from_numpy(x).to(d)
hi = torch.empty(x.shape, dtype=torch.int16, device=d)
lo = torch.empty_like(hi)
B.heal_split(xd, hi, lo)
st = status()
_, _, hb, lb = OS.split(x, OS.FP16_S11)
res["split_10001"] = {"status": st, "ok": st == B.HEAL_OK and
                      np.array_equal(hi.cpu().numpy().view(np.uint16), hb) and
                      np.array_equal(lo.cpu().numpy().view(np.uint16), lb)}

# INT16 KV writer into a larger cache at an offset
Qb, Kb, Vb = synthetic.kv_decode(B=2, T=70, Hkv=3, Hq=6, D=128, Tq=1, seeds=(5, 6, 7))
kc = torch.zeros(2, 3, 128, 128, dtype=torch.int16, device=d)
ks = torch.zeros(2, 3, 128, device=d)
B.heal_kv_quantize_int16(Kb.to(d), kc, ks, t_offset=40)
st = status()
qref, sref = OQ.quantize_kv(Kb.float().numpy())
res["kv_writer_offset"] = {"status": st, "ok": st == B.HEAL_OK and
                           np.array_equal(kc.cpu().numpy()[:, :, 40:110], qref) and
                           np.array_equal(ks.cpu().numpy()[:, :, 40:110].view(np.uint32), sref.view(np.uint32))}


def attention_case(name, Bt, Hq, Hkv, T, Tq, Tmax, kv_len, causal):
    Qb, Kb, Vb = synthetic.kv_decode(B=Bt, T=T, Hkv=Hkv, Hq=Hq, D=128, Tq=Tq, seeds=(11, 12, 13))
    q, qs = OQ.quantize_kv(Qb.float().numpy())
    kq, kss = OQ.quantize_kv(Kb.float().numpy())
    vq, vss = OQ.quantize_kv(Vb.float().numpy())
    pad = lambda a: np.concatenate([a, np.zeros(a.shape[:2] + (Tmax - T,) + a.shape[3:], a.dtype)], axis=2)
    kq, kss, vq, vss = pad(kq), pad(kss), pad(vq), pad(vss)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(d)
    out = torch.full((Bt, Hq, Tq, 128), float("nan"), device=d)
    ws = torch.empty(B.heal_attention_workspace_bytes(Bt, Hq, Tq, Tmax) // 4, device=d)
    hook = torch.full((Bt, Hq, Tq, Tmax), -1, dtype=torch.int64, device=d)
    B.heal_attention_int16(t(q), t(qs), t(kq), t(kss), t(vq), t(vss), t(np.asarray(kv_len, np.int32)), 128 ** -0.5,
                           out, ws, causal=causal, qk_int_out=hook)
    st = status()
    ref, s_blocks = OA.attention(q, qs, kq, kss, vq, vss, kv_len, 128 ** -0.5, causal=causal, return_s_int=True)
    o = out.cpu().numpy().astype(np.float64)
    h = hook.cpu().numpy()
    exact = True
    for b in range(Bt):
        L = int(kv_len[b])
        for i in range(Tq):
            vis = np.arange(L) <= (L - Tq + i) if causal else np.ones(L, bool)
            exact &= np.array_equal(h[b, :, i, :L][:, vis], s_blocks[b][:, i, :][:, vis])
    err = float(np.linalg.norm(o - ref) / np.linalg.norm(ref))
    res[name] = {"status": st, "err": err, "ok": st == B.HEAL_OK and exact and err <= 1e-4}


attention_case("attention_decode", 3, 8, 2, 200, 1, 256, [200, 77, 1], False)
attention_case("attention_prefill", 2, 8, 2, 190, 130, 192, [190, 150], True)

print(json.dumps(res))
