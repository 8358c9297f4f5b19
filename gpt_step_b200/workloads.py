"""Named workloads: model shapes, batch geometry, schedule and input recipe.

Shapes follow "Pretraining and adapting a language model on a dependency-free
stack" §4.1 and §4.4 (GPT-2 124M: 12 blocks, 12 heads, 768 channels, context
1,024, vocabulary 50,257 padded to 50,304; 19 sequences x 9 accumulation steps
per card) and the small-LM family table of grow_a_language_model_intro
("Eine Familie aus Drei": d_model 384 / 1536, vocabularies 4,353 / 8,449).
Pure data: no arithmetic of the method lives here.
"""

WORKLOADS = {
    "tiny": dict(n_layer=2, n_head=4, n_embd=128, seq_len=64, vocab_real=1000,
                 micro_batch=4, grad_accum=1, max_lr=6e-4, min_lr=0.0,
                 warmup_steps=0, total_steps=1, input="uniform", mean_doc_len=None,
                 seed=1337, steps=1),
    "small": dict(n_layer=6, n_head=12, n_embd=384, seq_len=1024, vocab_real=4353,
                  micro_batch=16, grad_accum=1, max_lr=6e-4, min_lr=0.0,
                  warmup_steps=5, total_steps=20, input="zipf", mean_doc_len=800,
                  seed=1337, steps=20),
    "gpt2_124m": dict(n_layer=12, n_head=12, n_embd=768, seq_len=1024, vocab_real=50257,
                      micro_batch=19, grad_accum=9, max_lr=6e-4, min_lr=0.0,
                      warmup_steps=700, total_steps=18865, input="zipf",
                      mean_doc_len=1000, seed=1337, steps=50),
    "gpt2_124m_b64": dict(n_layer=12, n_head=12, n_embd=768, seq_len=1024, vocab_real=50257,
                          micro_batch=64, grad_accum=8, max_lr=6e-4, min_lr=0.0,
                          warmup_steps=700, total_steps=18865, input="zipf",
                          mean_doc_len=1000, seed=1337, steps=50, eval_batches=20,
                          eval_batch=64, eval_seed=1338),
    "wide": dict(n_layer=16, n_head=24, n_embd=1536, seq_len=1024, vocab_real=8449,
                 micro_batch=8, grad_accum=8, max_lr=6e-4, min_lr=0.0,
                 warmup_steps=700, total_steps=18865, input="zipf", mean_doc_len=1000,
                 seed=1337, steps=30),
}

MODEL_KEYS = ("n_layer", "n_head", "n_embd", "seq_len", "vocab_real", "micro_batch",
              "grad_accum", "max_lr", "min_lr", "warmup_steps", "total_steps")


def model_args(name: str, **over) -> dict:
    w = dict(WORKLOADS[name])
    w.update(over)
    return {k: w[k] for k in MODEL_KEYS}
