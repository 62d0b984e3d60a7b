"""B200-native MLA decode attention over a paged latent KV cache (placeholder; binding follows)."""
