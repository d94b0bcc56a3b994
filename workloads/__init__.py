"""Seeded synthetic inputs for the MSA memory path (no method arithmetic lives here)."""
from .synth import CONFIGS, Config, get_config, gen_raw_slab, gen_query, gen_bank_bf16, doc_tok_offsets  # noqa: F401
