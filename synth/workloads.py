"""Workload shapes (model dimensions, batch, prompt and decode settings).

Each entry describes one synthetic workload: a random-init causal transformer
of a given shape plus the decode settings it runs with.  Weights are drawn by
``synth.weight_tensor``; prompts by ``synth.prompts``.

  tiny_f32        2-layer d128 fp32 model, B=1, P=16, N=32, W=4 (lambda 0.1, tau 0.5)
  tiny_f32_tau    same model with tau = 5.0 nats (about its median entropy), so the
                  threshold and multi-fill branches run
  qwen3_8b_b1     Qwen3-8B-shaped bf16 model, B=1, P=256, N=1024, W=16, lambda 0.1, tau 0.3
  qwen3_8b_b16    same model, B=16, P ~ U[128, 1024], N=1024, W=16, logit scale x{16, 4, 1}
  qwen25_7b_b64   Qwen2.5-7B-shaped bf16 model, B=64, P=8192, N=512, W=32,
                  lambda in {0, 0.05, 0.2} x tau in {0.1, 0.5}
  attn_micro      single-layer attention / selection microbench shapes
"""

QWEN3_8B = dict(L=36, d=4096, hq=32, hkv=8, hd=128, F=12288, V=151936, theta=1e6, eps=1e-6,
                mask_id=151935, dtype="bf16")
QWEN25_7B = dict(L=28, d=3584, hq=28, hkv=4, hd=128, F=18944, V=152064, theta=1e6, eps=1e-6,
                 mask_id=152063, dtype="bf16")
TINY = dict(L=2, d=128, hq=4, hkv=2, hd=32, F=384, V=512, theta=1e4, eps=1e-6, mask_id=511, dtype="f32")

CONFIGS = {
    "tiny_f32": dict(model=TINY, B=1, P=16, N=32, W=4, lam=0.1, tau=0.5, logit_scale=8.0, prompt_seed=1000),
    "tiny_f32_tau": dict(model=TINY, B=1, P=16, N=32, W=4, lam=0.1, tau=5.0, logit_scale=8.0, prompt_seed=1000),
    "attn_micro": dict(model=dict(L=1, d=4096, hq=32, hkv=8, hd=128, F=12288, V=151936, theta=1e6, eps=1e-6,
                                  mask_id=151935, dtype="bf16"),
                       B=(1, 2, 4, 8, 16, 32, 64), S=(1024, 4096, 16384, 32768), W=16, n_filled=8,
                       logit_std=(1.0, 4.0, 16.0), prompt_seed=1001),
    "qwen3_8b_b1": dict(model=QWEN3_8B, B=1, P=256, N=1024, W=16, lam=0.1, tau=0.3, logit_scale=1.0,
                        prompt_seed=1002),
    "qwen3_8b_b16": dict(model=QWEN3_8B, B=16, P=(128, 1024), N=1024, W=16, lam=0.1, tau=0.3,
                         logit_scale=4.0, logit_scales=(16.0, 4.0, 1.0), prompt_seed=1003),
    "qwen25_7b_b64": dict(model=QWEN25_7B, B=64, P=8192, N=512, W=32, lam=0.05, tau=0.5, logit_scale=1.0,
                          lams=(0.0, 0.05, 0.2), taus=(0.1, 0.5), prompt_seed=1004),
}


def model_dims(cfg: dict) -> dict:
    """The model-dimension dict of a workload (or the dict itself if it already is one)."""
    return cfg["model"] if "model" in cfg else cfg
