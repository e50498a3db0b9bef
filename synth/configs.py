"""Model shapes of the synthetic workloads (numbers only, no arithmetic).

Each dict uses the field names of the C ABI's ``dec_config``. Values the
source pages or the workload list leave open are filled with the pages'
defaults: RoPE base 10000, RMSNorm eps 1e-5, untied head unless stated,
no top-k renormalisation.
"""

COMMON = dict(qkv_bias=0, qk_norm=0, tied=0, n_experts=0, top_k=0, expert_inter=0,
              shared_inter=0, shared_gate=0, norm_topk=0, rms_eps=1e-5, rope_base=10000.0,
              page_size=16, prefill_chunk=128, max_batch=1, sliding_window=0, swa_pattern=0,
              attn_softcap=0.0, final_softcap=0.0, sandwich=0, weight_format=0)

# Tiny dense decoder: 16-token prompt then 8 greedy decode steps, batch 1.
TINY = dict(COMMON, name="tiny-dense", hidden=256, layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
            ffn_inter=688, vocab=1024, max_context=64)

# SmolLM2-135M shape: 1024-token prefill in chunks of 128, then batch-1 decode to 2048.
SMOLLM2_135M = dict(COMMON, name="smollm2-135m", hidden=576, layers=30, n_q_heads=9, n_kv_heads=3,
                    head_dim=64, ffn_inter=1536, vocab=49152, tied=1, max_context=2048)

# Llama-3-8B shape: decode at batch 1 and 32 at context 4096, 4096-token prefill in chunks of 128.
LLAMA3_8B = dict(COMMON, name="llama3-8b", hidden=4096, layers=32, n_q_heads=32, n_kv_heads=8,
                 head_dim=128, ffn_inter=14336, vocab=128256, rope_base=500000.0, max_context=4096,
                 max_batch=32)

# Qwen1.5-MoE-A2.7B shape: 60 routed experts (top-4 softmax), 1 sigmoid-gated shared expert,
# QKV bias; decode at batch 1 and 64 at context 2048.
QWEN15_MOE_A27B = dict(COMMON, name="qwen1.5-moe-a2.7b", hidden=2048, layers=24, n_q_heads=16,
                       n_kv_heads=16, head_dim=128, ffn_inter=0, vocab=151936, qkv_bias=1,
                       n_experts=60, top_k=4, expert_inter=1408, shared_inter=5632, shared_gate=1,
                       max_context=2048, max_batch=64)

# Standalone GQA decode-attention sweep.
GQA_SWEEP = dict(name="gqa-sweep", batch=64, n_q_heads=32, n_kv_heads=8, head_dim=128, page_size=16,
                 contexts=(512, 2048, 8192, 32768))

ALL = {c["name"]: c for c in (TINY, SMOLLM2_135M, LLAMA3_8B, QWEN15_MOE_A27B)}


def with_layers(cfg: dict, layers: int, **over) -> dict:
    """The same shape with fewer layers (a prefix of the full stack: same tensors, same ids)."""
    out = dict(cfg, layers=layers, **over)
    out["name"] = f"{cfg['name']}-L{layers}"
    return out
