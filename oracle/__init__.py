"""fp64 CPU oracle for one denoising step of sink-aware, query-predicted,
block-sparse bidirectional attention over a cached long-context KV.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this package: only tests/, the smoke check and the bench's CPU-baseline
leg may.  It shares no code with the CUDA library; both sides only read the
tensors drawn by the `synth` generator.

Every function is the plain definition of its step, written with numpy in
float64 (bf16/fp32 inputs convert to float64 exactly).  Softmax is two-pass
(row max, then sum of exponentials, then divide); there is no online
rescaling, no blocking and no fusion.  Ties in every top-k are broken by the
lower index, implemented as a stable sort on the negated value.

Sources (page title, then the part of the page):
  [F1] "Focus-dLLM: Accelerating Long-Context Diffusion LLM Inference via
       Confidence-Guided Context Focusing", abstract (chatpaper.ai, English
       abstract): past-confidence-guided indicator, sink-aware pruning, sink
       locations reused across layers, bidirectional full attention.
  [F2] same paper, research.elamur.ai summary and key points: previous-step
       confidence predicts the positions to unmask; guesses widened into
       local windows; predicted queries select the most relevant KV; sinks
       always kept and reused by deeper layers; shallow layers keep full
       attention; top-4 highest-confidence masked tokens (key point 1).
  [P1] "Prefilling-dLLM: Predictive Prefilling for Long-Context Inference in
       Diffusion Language Models", abstract (fugumt.com / aiqbench.com):
       prefix split into N chunks cached once, top-K chunks with
       intra-chunk token sparsity, a BOS token prepended to each chunk acts
       as a periodic attention anchor.
The pages give no formulas.  Where they are silent the readings below are
used (each is repeated at the function that applies it):
  R1 scale = 1/sqrt(d) for scoring and attention (standard scaled dot product).
  R2 block score = sum over predicted query rows (and over the query heads of
     a KV group) of that row's softmax over blocks of q . mean-pooled key.
  R3 selection is per KV head; sink blocks are excluded from the top-K
     candidates and then always added, so the count is K + |sink blocks|.
  R4 sink mass uses the predicted rows of every head, softmax over the whole
     context plus the decode block; one sink set per sequence.
  R5 windows are positional, clipped to the decode block; fewer masked
     positions than k means all of them are taken.
  R6 pooled keys are held at fp32, the precision the kernel stores them in:
     the exact fp64 mean is rounded once to fp32 and both sides score from
     those values (the selection decision is taken from the same pooled keys).
  R7 chunk path: chunk key = mean of its content tokens (BOS excluded); every
     decode query ranks chunks and tokens; the BOS of each selected chunk is
     always attended.
  R8 sinks are found once per decode block, at the first step's first sparse
     layer, and kept by every later step of the block: the pages keep sink
     locations consistent (reused across layers, and the cached context they
     index is unchanged until the block is written into the cache).
  R9 over head shards the sink mass is the sum of the shards' partial masses,
     each the R4 sum over that shard's heads only.
"""
from .steps import (  # noqa: F401
    scale_for, predict_queries, pool_mean, pooled_keys, block_scores,
    select_blocks, find_sinks, attention_rows, sparse_attention,
    gather_context, chunk_pooled_keys, chunk_scores, token_select,
    chunk_attention, dense_attention, topk_lower_index, cache_write,
)
from .step import (  # noqa: F401
    layer_step, chunked_step, denoise_block, StepResult, ChunkResult,
)
