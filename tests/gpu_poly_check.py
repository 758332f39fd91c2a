"""Run in a subprocess by test_gpu_parity: parity of one workload with the
exponential split chosen by STA_EXP_POLY8 (read once per process)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle.sta_oracle as O  # noqa: E402
import workloads as W  # noqa: E402
import sparse_attention_video_tile_b200 as sta  # noqa: E402


def main(name):
    cfg = W.CONFIGS[name]
    q, k, v = W.make_qkv(cfg, 5)
    out = sta.sta_forward(q.cuda(), k.cuda(), v.cuda(), cfg.grid, cfg.tile, cfg.windows, cfg.scale)
    assert sta.sta_check_device_status() == sta.STA_OK
    got = out.float().cpu().numpy()
    for h in range(cfg.heads):
        want = O.sta_attention_head(q[0, h].double().numpy(), k[0, h].double().numpy(), v[0, h].double().numpy(),
                                    cfg.grid, cfg.tile, cfg.windows[h], cfg.scale)
        err = np.abs(got[0, h] - want).max()
        rel = np.linalg.norm(got[0, h] - want) / np.linalg.norm(want)
        if not (err <= 1e-2 and rel <= 5e-3):
            print(f"head {h}: max abs {err:.3e} rel {rel:.3e}")
            return 1
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1]))
