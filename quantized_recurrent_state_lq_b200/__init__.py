"""quantized_recurrent_state_lq_b200: windowed INT8 recurrent-state decode for B200."""
