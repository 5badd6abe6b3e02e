"""Runs the layer's kernels once through whichever library _lib loads (TG_DEBUG=1 in
the environment: the debug library) and saves every output and the device status
word to the path given on the command line. tests/test_gpu_debug_build.py runs it
twice, once per library, and compares the two files bit for bit."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from learned_token_pruning_gemm_b200 import _lib, api, pipeline, synth  # noqa: E402


def main(path):
    lib = _lib.load()
    res = {"debug_build": int(lib.tg_debug_build())}
    api.device_status(reset=True)
    # the layer, bf16 with the kept rows' projections on a ragged batch, and fp32
    for name, proj, fuse in (("ragged8", True, False), ("ragged8_fused", True, True),
                             ("tiny_f32", False, False)):
        wl = synth.WORKLOADS[name.replace("_fused", "")]()
        gp = pipeline.GatedPrefill(wl, project=proj, fuse=fuse)
        gp.step()
        torch.cuda.synchronize()
        for attr in ("scores", "kept_idx", "kept_scores", "cu_kept", "kept_pos", "xc", "q", "k",
                     "v", "out"):
            t = getattr(gp, attr, None)
            if t is not None:
                res[f"{name}.{attr}"] = t.cpu()
        if name == "ragged8":
            # the Gated DeltaNet rule over the same kept rows
            q, k, v, a, b = synth.deltanet_inputs(wl)
            res["deltanet"] = api.gated_delta_rule(q.cuda(), k.cuda(), v.cuda(), a.cuda(),
                                                   b.cuda(), gp.cu_kept).cpu()
    # the backward of the gated attention on a ragged batch, bf16 and fp32
    g = torch.Generator().manual_seed(3)
    for dt, lens in ((torch.bfloat16, [300, 1, 129, 700]), (torch.float32, [37, 1, 90])):
        K, hq, hkv = sum(lens), 16, 8
        dh = 128 if dt == torch.bfloat16 else 64
        q = torch.randn(K, hq, dh, generator=g).to(dt).cuda()
        k = torch.randn(K, hkv, dh, generator=g).to(dt).cuda()
        v = torch.randn(K, hkv, dh, generator=g).to(dt).cuda()
        do = torch.randn(K, hq, dh, generator=g).to(dt).cuda()
        s = (torch.randn(K, generator=g) * 2).cuda()
        gain = torch.rand(hq, generator=g).cuda()
        tau = (0.8 + 0.7 * torch.rand(hq, generator=g)).cuda()
        cu = torch.tensor(np.r_[0, np.cumsum(lens)].astype(np.int32), device="cuda")
        lse = torch.empty(hq, K, device="cuda")
        out = api.gated_attention(q, k, v, s, gain, tau, cu, max(lens), lse=lse)
        grads = api.gated_attention_bwd(q, k, v, out, do, lse, s, gain, tau, cu, max(lens))
        res[f"bwd_{dt}.out"] = out.cpu()
        res[f"bwd_{dt}.lse"] = lse.cpu()
        for i, t in enumerate(grads):
            res[f"bwd_{dt}.{i}"] = t.cpu()
    # decode over a ragged cache: append a token, then attend
    B, cap, lens, hq, hkv = 3, 700, [699, 129, 1], 16, 8
    qd = torch.randn(B, hq, 128, generator=g).to(torch.bfloat16).cuda()
    kc = torch.randn(B, cap, hkv, 128, generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn(B, cap, hkv, 128, generator=g).to(torch.bfloat16).cuda()
    sc = (torch.randn(B, cap, generator=g) * 2).cuda()
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    gain = torch.rand(hq, generator=g).cuda()
    tau = (0.8 + 0.7 * torch.rand(hq, generator=g)).cuda()
    kn = torch.randn(B, hkv, 128, generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn(B, hkv, 128, generator=g).to(torch.bfloat16).cuda()
    sn = torch.randn(B, generator=g).cuda()
    api.cache_append(kn, vn, sn, kc, vc, sc, ln)
    res["decode"] = api.gated_decode(qd, kc, vc, sc, ln, gain, tau, cap).cpu()
    res["decode.kc"] = kc.cpu()
    res["decode.len"] = ln.cpu()
    torch.cuda.synchronize()
    res["status"] = int(api.device_status(reset=True))
    torch.save(res, path)


if __name__ == "__main__":
    main(sys.argv[1])
