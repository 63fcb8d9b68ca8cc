"""latent_kv_attention_b200 -- grouped / latent-KV attention for B200 (sm_100a)."""
