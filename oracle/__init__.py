"""Float64 CPU oracle of the routed-expert MoE prefill layer (test infrastructure only)."""
