"""Small standalone workloads for kernel profiling (one call each, synthetic inputs).

    python -m token_sparse_long_b200.profile_case score --S 16384 --H 32 --blk 128
    python -m token_sparse_long_b200.profile_case layer --S 16384 --keep 0.5

`score` runs jenga_score_blocks on random bf16 q, k ([S, H*128], N(0, 0.3)); `layer` runs one
7B-shaped layer (hidden 4096, 32 heads, FFN 11008) at the given length: q/k of all rows,
scoring, top-k selection, the retained-token forward and backward (segments of 4096).
Each runs its path twice (the second call is the one a profiler should capture)."""
import argparse

import torch


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["score", "layer", "blockmax"])
    ap.add_argument("--S", type=int, default=16384)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--blk", type=int, default=128)
    ap.add_argument("--keep", type=float, default=0.5)
    a = ap.parse_args()
    import token_sparse_long_b200 as J
    J._lib.load()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    if a.what in ("score", "blockmax"):
        q = (torch.randn(a.S, a.H * 128, device=dev, generator=g) * 0.3).to(torch.bfloat16)
        k = (torch.randn(a.S, a.H * 128, device=dev, generator=g) * 0.3).to(torch.bfloat16)
        mode = "softmax_mass" if a.what == "score" else "paper_blockmax"
        for _ in range(2):
            J.jenga_score_blocks(q, k, a.H, 128, a.blk, mode=mode)
    else:
        h, F, H = 4096, 11008, 32
        n = lambda *s: (torch.randn(*s, device=dev, generator=g) * 0.02).to(torch.bfloat16)  # noqa: E731
        ones = torch.ones(h, device=dev, dtype=torch.bfloat16)
        L = J.LayerHandle(n(H * 128, h), n(H * 128, h), n(H * 128, h), n(h, H * 128), n(F, h), n(F, h), n(h, F), ones,
                          ones.clone(), n(16, h), n(H * 128, 16), n(16, h), n(H * 128, 16), heads=H, head_dim=128)
        x0 = torch.randn(a.S, h, device=dev, generator=g).to(torch.bfloat16)
        g0 = torch.randn(a.S, h, device=dev, generator=g).to(torch.bfloat16)
        nb = a.S // a.blk
        kmax = max(1, int(-(-a.keep * nb // 1)))
        for _ in range(2):
            x = x0.clone()
            qk = J.jenga_layer_score_qk(L, x)
            sc = J.jenga_score_blocks(qk[:, :H * 128], qk[:, H * 128:], H, 128, a.blk)
            idx, nk, _ = J.jenga_select(sc, "topk", kmax)
            saved = J.jenga_sparse_layer_fwd(L, x, idx, nk, a.blk, kmax, qk=qk)
            dx = g0.clone()
            J.jenga_sparse_layer_bwd(L, dx, idx, nk, a.blk, kmax, saved, J.new_lora_grads(L), segment_tokens=4096)
    J.jenga_check_device_status()
    torch.cuda.synchronize()
    print("ok")


if __name__ == "__main__":
    main()
